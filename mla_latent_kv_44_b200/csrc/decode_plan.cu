// Split-KV schedule and log-sum-exp combine of mla_decode.
//
// Every (sequence b, query token t) row group attends L = seq_lens[b] - T + 1 + t rows; its
// rows are cut into 64-row chunks and all chunks of the call are laid end to end. The planner
// cuts that list into R = min(74, chunks) ranges of equal size (range q starts at chunk
// floor(q * C / R)). A row group touched by one range is a single segment whose result goes
// straight to the output; a row group crossed by range boundaries becomes several segments
// whose softmax-normalised partial results (with their log-sum-exp) are merged by the combine
// kernel. Integer work only: the schedule is a pure function of seq_lens.
#include "plan_body.cuh"

namespace mla {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(DecodeParams p) {
  __shared__ int s_a[32], s_b[32], s_carry[2];
  plan_body<kPlanThreads>(p, s_a, s_b, s_carry);
}

cudaError_t launch_plan(const DecodeParams& p, cudaStream_t st) {
  return launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, p);
}

// ------------------------------------------------------------------------------------------
// Combine: out = sum_i exp(lse_i - L) * o_i, L = log sum_i exp(lse_i), in segment order.
// One CTA per (row group, 4 heads), one warp per head. Row groups with a single segment were
// written directly by the attention kernel and are skipped; row groups with an invalid length
// get 0 and -inf. The weights exp(lse_i - L) are computed once per (row group, head) into
// shared memory; the partial rows are then streamed as float4 (a lane holds 4 of the r dims).
// ------------------------------------------------------------------------------------------
constexpr int kCombineHeads = 4;

__global__ void __launch_bounds__(kCombineHeads * 32) combine_kernel(DecodeParams p) {
  __shared__ float s_w[kCombineHeads][kRanges];
  const int bt = blockIdx.x;
  wait_prior_grid();
  const int nseg = p.bt_nseg[bt];
  const int slot0 = p.bt_slot0[bt];  // a split row group's slots are slot0 .. slot0 + nseg - 1
  if (nseg == 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kCombineHeads + warp;
  if (h >= p.H) return;
  float4* dst = (float4*)(p.out + ((size_t)bt * p.H + h) * p.r);
  const int r4 = p.r / 4;
  const float L = merge_weights(p, slot0, nseg, h, s_w[warp]);
  if (L == -INFINITY) {  // no rows (bad length, or every block rejected)
    for (int d = lane; d < r4; d += 32) dst[d] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0 && p.lse) p.lse[(size_t)bt * p.H + h] = -INFINITY;
    return;
  }
  // a lane holds up to four float4 of the row at once (r = 512 in one pass), so every partial's
  // loads for the whole row are in flight together
  for (int d0 = lane; d0 < r4; d0 += 128) {
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int k = 0; k < nseg; ++k) {
      const float w = s_w[warp][k];
      const float4* src = (const float4*)(p.part_o + ((size_t)(slot0 + k) * p.H + h) * p.r);
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = (d0 + 32 * u < r4) ? __ldcs(src + d0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[u].x = fmaf(w, v[u].x, acc[u].x);
        acc[u].y = fmaf(w, v[u].y, acc[u].y);
        acc[u].z = fmaf(w, v[u].z, acc[u].z);
        acc[u].w = fmaf(w, v[u].w, acc[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (d0 + 32 * u < r4) dst[d0 + 32 * u] = acc[u];
  }
  if (lane == 0 && p.lse) p.lse[(size_t)bt * p.H + h] = L;
}

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t st) {
  dim3 grid(p.BT, (p.H + kCombineHeads - 1) / kCombineHeads);
  return launch_pdl(combine_kernel, grid, dim3(128), 0, st, p);
}

// ------------------------------------------------------------------------------------------
// Merge of results computed apart: `parts` softmax-normalised partial results of the same n
// row groups over disjoint sets of cache rows (one per GPU of a context-parallel split of
// every sequence's rows), laid out part-major: o (parts, n, H, r), lse (parts, n, H). The
// same log-sum-exp merge as above, in part order. A part with lse = -inf holds no rows and is
// skipped whatever its o; a row group with no rows in any part gets 0 and -inf.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kCombineHeads * 32)
combine_parts_kernel(const float* part_o, const float* part_lse, int parts, int n, int H, int r,
                     float* out, float* lse) {
  __shared__ float s_w[kCombineHeads][MLA_MAX_COMBINE_PARTS];
  wait_prior_grid();
  const int bt = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kCombineHeads + warp;
  if (h >= H) return;
  const size_t plane = (size_t)n * H;  // one part's (n, H) entries
  const size_t at = (size_t)bt * H + h;
  float mx = -INFINITY;
  for (int k = lane; k < parts; k += 32) mx = fmaxf(mx, part_lse[k * plane + at]);
  mx = warp_max(mx);
  float4* dst = (float4*)(out + at * r);
  const int r4 = r / 4;
  if (mx == -INFINITY) {
    for (int d = lane; d < r4; d += 32) dst[d] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0 && lse) lse[at] = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = lane; k < parts; k += 32) z += expf(part_lse[k * plane + at] - mx);
  z = warp_sum(z);
  const float L = mx + logf(z);
  for (int k = lane; k < parts; k += 32) s_w[warp][k] = expf(part_lse[k * plane + at] - L);
  __syncwarp();
  for (int d0 = lane; d0 < r4; d0 += 128) {
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < parts; ++k) {
      const float w = s_w[warp][k];
      if (w == 0.f) continue;  // an empty part (or one far below the others)
      const float4* src = (const float4*)(part_o + (k * plane + at) * r);
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = (d0 + 32 * u < r4) ? __ldcs(src + d0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[u].x = fmaf(w, v[u].x, acc[u].x);
        acc[u].y = fmaf(w, v[u].y, acc[u].y);
        acc[u].z = fmaf(w, v[u].z, acc[u].z);
        acc[u].w = fmaf(w, v[u].w, acc[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (d0 + 32 * u < r4) dst[d0 + 32 * u] = acc[u];
  }
  if (lane == 0 && lse) lse[at] = L;
}

cudaError_t launch_combine_parts(const float* part_o, const float* part_lse, int parts, int n,
                                 int H, int r, float* out, float* lse, cudaStream_t st) {
  dim3 grid(n, (H + kCombineHeads - 1) / kCombineHeads);
  return launch_pdl(combine_parts_kernel, grid, dim3(kCombineHeads * 32), 0, st, part_o,
                    part_lse, parts, n, H, r, out, lse);
}

}  // namespace mla
