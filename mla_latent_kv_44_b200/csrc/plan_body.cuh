// The decode planner's body and the log-sum-exp merge weights, shared by the kernels of
// mla_decode (decode_plan.cu) and the fused step kernels (proj_tc.cu).
//
// Every (sequence b, query token t) row group attends L = seq_lens[b] - T + 1 + t rows; its
// rows are cut into 64-row chunks and all chunks of the call are laid end to end. The planner
// cuts that list into R = min(74, chunks) ranges of equal size (range q starts at chunk
// floor(q * C / R)). A row group touched by one range is a single segment whose result goes
// straight to the output; a row group crossed by range boundaries becomes several segments
// whose softmax-normalised partial results (with their log-sum-exp) are merged afterwards.
// Integer work only: the schedule is a pure function of seq_lens.
#pragma once

#include "common.cuh"

namespace mla {

// Number of range starts strictly below chunk x: #{q in [0,R) : floor(q*C/R) < x}.
__device__ __forceinline__ int starts_below(int64_t x, int64_t R, int64_t C) {
  if (x <= 0 || C <= 0) return 0;
  const int64_t v = (x * R + C - 1) / C;
  return (int)(v < R ? v : R);
}

__device__ __forceinline__ int range_start(int64_t q, int64_t R, int64_t C) {
  return (int)((q * C) / R);
}

// Inclusive block scan of two ints over NT threads (NT a multiple of 32, at most 1024):
// shuffle scans inside each warp, then the first warp scans the warp totals. s_a / s_b hold at
// least 32 ints.
template <int NT>
__device__ void block_scan2(int* s_a, int* s_b, int& a, int& b) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps, at most 32 of them");
  constexpr int kWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, a, o), vb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += va;
      b += vb;
    }
  }
  if (lane == 31) {
    s_a[warp] = a;
    s_b[warp] = b;
  }
  __syncthreads();
  if (warp == 0) {
    int wa = lane < kWarps ? s_a[lane] : 0, wb = lane < kWarps ? s_b[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int va = __shfl_up_sync(0xffffffffu, wa, o), vb = __shfl_up_sync(0xffffffffu, wb, o);
      if (lane >= o) {
        wa += va;
        wb += vb;
      }
    }
    if (lane < kWarps) {
      s_a[lane] = wa;
      s_b[lane] = wb;
    }
  }
  __syncthreads();
  if (warp > 0) {
    a += s_a[warp - 1];
    b += s_b[warp - 1];
  }
  __syncthreads();  // s_a / s_b are reused by the next scan
}

// The planner, run by one CTA of NT threads (s_a, s_b: at least 32 ints of shared memory each;
// carry: two ints). Waits for the previous grid before it reads seq_lens.
template <int NT>
__device__ void plan_body(const DecodeParams& p, int* s_a, int* s_b, int* carry) {
  constexpr int kPlanThreads = NT;
  int& s_carry_a = carry[0];
  int& s_carry_b = carry[1];
  const int tid = threadIdx.x;
  const int64_t cap = (int64_t)p.max_blocks * p.bs;
  wait_prior_grid();

  // Pass 1: attended lengths, chunk counts, exclusive prefix of chunk counts. With at most
  // kPlanThreads row groups (one pass), pass 2 takes them from registers.
  int my_len = 0, my_chunk0 = 0;
  if (tid == 0) s_carry_a = 0;
  __syncthreads();
  for (int base = 0; base < p.BT; base += kPlanThreads) {
    const int bt = base + tid;
    int nch = 0;
    if (bt < p.BT) {
      const int b = bt / p.T, t = bt - b * p.T;
      const int sl = p.seq_lens[b];
      int len = 0;
      if (sl < p.T || (int64_t)sl > cap) {
        if (t == 0) set_error(p.err, MLA_DEV_BAD_LENGTH);
      } else {
        len = sl - p.T + 1 + t;
      }
      nch = (len + kChunk - 1) / kChunk;
      p.bt_len[bt] = len;
      my_len = len;
    }
    int inc = nch, dummy = 0;
    block_scan2<NT>(s_a, s_b, inc, dummy);
    if (bt < p.BT) {
      my_chunk0 = s_carry_a + inc - nch;
      p.bt_chunk0[bt] = my_chunk0;
    }
    __syncthreads();
    if (tid == kPlanThreads - 1) s_carry_a += inc;
    __syncthreads();
  }
  const int C = s_carry_a;
  const int R = C < kRanges ? C : kRanges;
  __syncthreads();

  // Pass 2: segments per row group, their global indices and partial-result slots.
  if (tid == 0) { s_carry_a = 0; s_carry_b = 0; }
  __syncthreads();
  for (int base = 0; base < p.BT; base += kPlanThreads) {
    const int bt = base + tid;
    int nseg = 0, nslot = 0, x = 0, e = 0;
    if (bt < p.BT) {
      const bool one_pass = p.BT <= kPlanThreads;
      const int len = one_pass ? my_len : p.bt_len[bt];
      const int nch = (len + kChunk - 1) / kChunk;
      x = one_pass ? my_chunk0 : p.bt_chunk0[bt];
      e = x + nch;
      if (nch > 0) nseg = 1 + starts_below(e, R, C) - starts_below(x + 1, R, C);
      nslot = nseg >= 2 ? nseg : 0;
    }
    int inc_seg = nseg, inc_slot = nslot;
    block_scan2<NT>(s_a, s_b, inc_seg, inc_slot);
    if (bt < p.BT) {
      const int first = s_carry_a + inc_seg - nseg;
      const int slot0 = s_carry_b + inc_slot - nslot;
      p.bt_slot0[bt] = nseg >= 2 ? slot0 : -1;
      p.bt_nseg[bt] = nseg;
      // cut points of this row group: x, the range starts strictly inside (x, e), e
      int q = starts_below(x + 1, R, C);  // first range starting after x
      int lo = x;
      for (int k = 0; k < nseg; ++k) {
        const int hi = (k == nseg - 1) ? e : range_start(q, R, C);
        Segment sg;
        sg.bt = bt;
        sg.chunk_lo = lo;
        sg.chunk_hi = hi;
        sg.slot = nseg >= 2 ? slot0 + k : -1;
        p.segments[first + k] = sg;
        // a range starting exactly here begins with this segment
        const int qs = starts_below(lo + 1, R, C) - 1;  // range containing chunk lo
        if (qs >= 0 && range_start(qs, R, C) == lo) p.range_begin[qs] = first + k;
        lo = hi;
        ++q;
      }
    }
    __syncthreads();
    if (tid == kPlanThreads - 1) { s_carry_a += inc_seg; s_carry_b += inc_slot; }
    __syncthreads();
  }
  if (tid == 0) {
    p.header[0] = s_carry_a;  // segments
    p.header[1] = R;          // ranges in use
    p.header[2] = C;          // chunks
    p.range_begin[R] = s_carry_a;
  }
}


// Weights of a split row group's partial results for head h, computed by one warp:
// w[k] = exp(lse_k - L) for its nseg slots (into shared memory), L = log sum_k exp(lse_k).
// Returns L; returns -inf (and writes no weight) when there are no rows (nseg == 0 or every
// partial empty). The sums run in the same order wherever this is called, so every merge of
// the same partials gives the same bits.
__device__ __forceinline__ float merge_weights(const DecodeParams& p, int slot0, int nseg, int h,
                                               float* w) {
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  for (int k = lane; k < nseg; k += 32) mx = fmaxf(mx, p.part_lse[(size_t)(slot0 + k) * p.H + h]);
  mx = warp_max(mx);
  if (nseg == 0 || mx == -INFINITY) return -INFINITY;
  float z = 0.f;
  for (int k = lane; k < nseg; k += 32) z += expf(p.part_lse[(size_t)(slot0 + k) * p.H + h] - mx);
  z = warp_sum(z);
  const float L = mx + logf(z);
  for (int k = lane; k < nseg; k += 32) w[k] = expf(p.part_lse[(size_t)(slot0 + k) * p.H + h] - L);
  __syncwarp();
  return L;
}

}  // namespace mla
