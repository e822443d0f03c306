// CUDA-core attention stage of mla_decode (any shape; fp32, bf16 or fp8 e4m3 rows with a
// per-row scale; fp32 math).
//
// Absorbed form ("DeepSeek MLA, Built From the Paper", 3 Matrix absorption; "MLA from scratch
// in PyTorch", Absorbing projections): each head scores the packed query [q_lat || q_rope]
// against whole cached rows [c_kv || k_rope] and accumulates the softmax-weighted c_kv part.
//
// One CTA per (segment, group of 8 heads); warp w owns head 8*blockIdx.y + w. Rows are staged
// 32 at a time in shared memory as fp32 with an odd word stride, so that lane t computing the
// score of row t and all lanes reading one row are both bank-conflict free. Online softmax in
// fp32 (running max m, running sum l), exact exp, fixed summation order: deterministic.
#include <cuda_fp8.h>

#include "common.cuh"

namespace mla {

// an fp8 (e4m3) cache code
struct Fp8Code {
  uint8_t bits;
};

constexpr int kSimtHeads = 8;   // warps (heads) per CTA
constexpr int kSimtRows = 32;   // rows per staged tile (one per lane)

// e4m3 code -> float (exact: every e4m3 value is a half)
__device__ __forceinline__ float fp8_to_f32(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}

// TQ: the query's type, TR: the rows' (Fp8Code: codes times the row's scale)
template <typename TQ, typename TR, int RW>  // RW: latent columns per lane (r <= 32 * RW)
__global__ void __launch_bounds__(kSimtHeads * 32)
attend_simt_kernel(DecodeParams p) {
  const int seg_id = blockIdx.x;
  wait_prior_grid();
  if (seg_id >= p.header[0]) return;
  const Segment sg = p.segments[seg_id];
  const int bt = sg.bt, b = bt / p.T;
  const int len = p.bt_len[bt];
  const int chunk0 = p.bt_chunk0[bt];  // segment chunks are numbered across all row groups
  const int tok_lo = (sg.chunk_lo - chunk0) * kChunk;
  const int tok_hi = min((sg.chunk_hi - chunk0) * kChunk, len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kSimtHeads + warp;
  const bool active = h < p.H;
  const int D = p.D, ld = D + 1, r = p.r;

  extern __shared__ float smem[];
  float* s_rows = smem;                          // kSimtRows x ld
  float* s_q = smem + kSimtRows * ld;            // kSimtHeads x D
  int* s_ok = (int*)(s_q + kSimtHeads * D);      // kSimtRows
  float* s_scale = (float*)(s_ok + kSimtRows);   // kSimtRows (fp8 rows)

  const TQ* Q = (const TQ*)p.q;
  const TR* pool = (const TR*)p.pool;
  for (int idx = threadIdx.x; idx < kSimtHeads * D; idx += blockDim.x) {
    const int hh = blockIdx.y * kSimtHeads + idx / D;
    s_q[idx] = hh < p.H ? to_f32(Q[((size_t)bt * p.H + hh) * D + idx % D]) : 0.f;
  }

  float o[RW];
#pragma unroll
  for (int k = 0; k < RW; ++k) o[k] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int quads = D / 4;

  for (int t0 = tok_lo; t0 < tok_hi; t0 += kSimtRows) {
    __syncthreads();  // previous tile fully consumed (and s_q written on the first pass)
    if (threadIdx.x < kSimtRows) {
      const int tok = t0 + threadIdx.x;
      int ok = 0;
      if (tok < tok_hi) {
        const int blk = p.table[(size_t)b * p.max_blocks + tok / p.bs];
        if (blk >= 0 && blk < p.num_blocks) ok = 1 + blk;  // store block id + 1
        else set_error(p.err, MLA_DEV_OOB_BLOCK);
      }
      s_ok[threadIdx.x] = ok;
      if (sizeof(TR) == 1)
        s_scale[threadIdx.x] = ok ? p.row_scale[(size_t)(ok - 1) * p.bs + tok % p.bs] : 0.f;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kSimtRows * quads; idx += blockDim.x) {
      const int t = idx / quads, qd = idx - t * quads;
      const int ok = s_ok[t];
      float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
      if (ok) {
        const int tok = t0 + t;
        const TR* row = pool + ((size_t)(ok - 1) * p.bs + tok % p.bs) * D + 4 * qd;
        if (sizeof(TR) == 4) {
          const float4 v = *(const float4*)row;
          v0 = v.x; v1 = v.y; v2 = v.z; v3 = v.w;
        } else if (sizeof(TR) == 1) {
          const uint32_t u = *(const uint32_t*)row;
          const float sc = s_scale[t];
          v0 = fp8_to_f32(u & 0xffu) * sc;
          v1 = fp8_to_f32((u >> 8) & 0xffu) * sc;
          v2 = fp8_to_f32((u >> 16) & 0xffu) * sc;
          v3 = fp8_to_f32(u >> 24) * sc;
        } else {
          const uint2 u = *(const uint2*)row;
          const __nv_bfloat162 a = *(const __nv_bfloat162*)&u.x;
          const __nv_bfloat162 c = *(const __nv_bfloat162*)&u.y;
          v0 = __low2float(a); v1 = __high2float(a); v2 = __low2float(c); v3 = __high2float(c);
        }
      }
      float* dst = s_rows + t * ld + 4 * qd;
      dst[0] = v0; dst[1] = v1; dst[2] = v2; dst[3] = v3;
    }
    __syncthreads();
    if (!active) continue;

    // score of row t0 + lane
    float s = -INFINITY;
    if (s_ok[lane]) {
      const float* qrow = s_q + warp * D;
      const float* krow = s_rows + lane * ld;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = fmaf(qrow[d], krow[d], acc);
      s = acc * p.scale;
    }
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;  // nothing valid yet
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float pe = (s == -INFINITY) ? 0.f : expf(s - m_new);
    l = l * alpha + warp_sum(pe);
#pragma unroll
    for (int k = 0; k < RW; ++k) o[k] *= alpha;
    for (int t = 0; t < kSimtRows; ++t) {
      const float pt = __shfl_sync(0xffffffffu, pe, t);
      const float* row = s_rows + t * ld;
#pragma unroll
      for (int k = 0; k < RW; ++k) {
        const int d = lane + 32 * k;
        if (d < r) o[k] = fmaf(pt, row[d], o[k]);
      }
    }
    m = m_new;
  }
  if (!active) return;
  const bool empty = (l == 0.f);
  const float inv = empty ? 0.f : 1.f / l;
  const float lse = empty ? -INFINITY : m + logf(l);
  float* dst;
  if (sg.slot < 0) {
    dst = p.out + ((size_t)bt * p.H + h) * r;
    if (lane == 0 && p.lse) p.lse[(size_t)bt * p.H + h] = lse;
  } else {
    dst = p.part_o + ((size_t)sg.slot * p.H + h) * r;
    if (lane == 0) p.part_lse[(size_t)sg.slot * p.H + h] = lse;
  }
#pragma unroll
  for (int k = 0; k < RW; ++k) {
    const int d = lane + 32 * k;
    if (d < r) dst[d] = o[k] * inv;
  }
}

template <typename TQ, typename TR, int RW>
static cudaError_t simt_go(const DecodeParams& p, cudaStream_t st) {
  const size_t smem = sizeof(float) * (kSimtRows * (p.D + 1) + kSimtHeads * p.D) +
                      (sizeof(int) + sizeof(float)) * kSimtRows;
  auto k = attend_simt_kernel<TQ, TR, RW>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(kRanges + p.BT, (p.H + kSimtHeads - 1) / kSimtHeads);
  return launch_pdl(k, grid, dim3(kSimtHeads * 32), smem, st, p);
}

template <typename TQ, typename TR>
static cudaError_t simt_dispatch(const DecodeParams& p, cudaStream_t st) {
  if (p.r <= 64) return simt_go<TQ, TR, 2>(p, st);
  if (p.r <= 128) return simt_go<TQ, TR, 4>(p, st);
  if (p.r <= 256) return simt_go<TQ, TR, 8>(p, st);
  if (p.r <= 512) return simt_go<TQ, TR, 16>(p, st);
  return simt_go<TQ, TR, 32>(p, st);
}

cudaError_t launch_attend_simt(const mla_config& c, const DecodeParams& p, cudaStream_t st) {
  return c.dtype == MLA_BF16 ? simt_dispatch<__nv_bfloat16, __nv_bfloat16>(p, st)
                             : simt_dispatch<float, float>(p, st);
}

cudaError_t launch_attend_simt_fp8(const mla_config& c, const DecodeParams& p, cudaStream_t st) {
  return c.dtype == MLA_BF16 ? simt_dispatch<__nv_bfloat16, Fp8Code>(p, st)
                             : simt_dispatch<float, Fp8Code>(p, st);
}

}  // namespace mla
