// Per-token kernels of the MLA decode step: absorbed query, cache append, output projection.
//
// Sources: "DeepSeek MLA, Built From the Paper", 3 Matrix absorption (W_UK folds into the
// query); "MLA from scratch in PyTorch", The MLAAttention module (norm_kv before caching) and
// Absorbing projections (W_UV after the weighted sum); "Multi-head latent attention",
// Compress keys and values into one latent (row = [c_kv || k_rope], k_rope shared by heads).
#include "append_row.cuh"

namespace mla {

// ------------------------------------------------------------------------------------------
// Absorbed query: Q[n,h,:r] = W_UK[h]^T q_nope[n,h];  Q[n,h,r:] = RoPE(q_rope[n,h], pos[n]).
// One CTA per (16 tokens, head); thread j owns latent columns j, j+256, ... of W_UK[h], which
// it streams row by row (coalesced across the CTA) while the 16 query rows sit in shared memory.
// ------------------------------------------------------------------------------------------
constexpr int kAbsorbTokens = 16;

template <typename T, int COLS>
__global__ void __launch_bounds__(256)
absorb_kernel(const T* __restrict__ q_nope, const T* __restrict__ q_rope,
              const int32_t* __restrict__ pos, const T* __restrict__ w_uk, T* __restrict__ q_out,
              int n, int H, int dh, int r, int dr, float base) {
  extern __shared__ float s_q[];  // kAbsorbTokens x dh
  wait_prior_grid();
  const int h = blockIdx.y;
  const int n0 = blockIdx.x * kAbsorbTokens;
  const int nt = min(kAbsorbTokens, n - n0);
  for (int idx = threadIdx.x; idx < kAbsorbTokens * dh; idx += blockDim.x) {
    const int t = idx / dh, i = idx - t * dh;
    s_q[idx] = t < nt ? to_f32(q_nope[((size_t)(n0 + t) * H + h) * dh + i]) : 0.f;
  }
  __syncthreads();

  float acc[kAbsorbTokens][COLS];
#pragma unroll
  for (int t = 0; t < kAbsorbTokens; ++t)
#pragma unroll
    for (int c = 0; c < COLS; ++c) acc[t][c] = 0.f;

  const T* W = w_uk + (size_t)h * dh * r;
  for (int i = 0; i < dh; ++i) {
    float wv[COLS];
#pragma unroll
    for (int c = 0; c < COLS; ++c) {
      const int j = threadIdx.x + c * 256;
      wv[c] = j < r ? to_f32(W[(size_t)i * r + j]) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < kAbsorbTokens; ++t) {
      const float qv = s_q[t * dh + i];
#pragma unroll
      for (int c = 0; c < COLS; ++c) acc[t][c] = fmaf(qv, wv[c], acc[t][c]);
    }
  }
  const int D = r + dr;
#pragma unroll
  for (int t = 0; t < kAbsorbTokens; ++t) {
    if (t >= nt) break;
    T* dst = q_out + ((size_t)(n0 + t) * H + h) * D;
#pragma unroll
    for (int c = 0; c < COLS; ++c) {
      const int j = threadIdx.x + c * 256;
      if (j < r) dst[j] = from_f32<T>(acc[t][c]);
    }
  }
  // RoPE part of the query (pairs (2i, 2i+1), angle pos * base^(-2i/dr) in double).
  const int half = dr / 2;
  for (int idx = threadIdx.x; idx < nt * half; idx += blockDim.x) {
    const int t = idx / half, i = idx - t * half;
    double c, s;
    rope_cos_sin(pos[n0 + t], i, dr, base, &c, &s);
    const T* src = q_rope + ((size_t)(n0 + t) * H + h) * dr;
    const double x0 = to_f32(src[2 * i]), x1 = to_f32(src[2 * i + 1]);
    T* dst = q_out + ((size_t)(n0 + t) * H + h) * D + r;
    dst[2 * i] = from_f32<T>((float)(x0 * c - x1 * s));
    dst[2 * i + 1] = from_f32<T>((float)(x0 * s + x1 * c));
  }
}

template <typename T, int COLS>
static cudaError_t absorb_go(const mla_config& c, const void* qn, const void* qr,
                             const int32_t* pos, const void* w, void* q, int n, cudaStream_t st) {
  const size_t smem = sizeof(float) * kAbsorbTokens * c.head_dim;
  auto k = absorb_kernel<T, COLS>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((n + kAbsorbTokens - 1) / kAbsorbTokens, c.num_heads);
  return launch_pdl(k, grid, dim3(256), smem, st, (const T*)qn, (const T*)qr, pos, (const T*)w,
                    (T*)q, n, c.num_heads, c.head_dim, c.kv_rank, c.rope_dim, c.rope_base);
}

template <typename T>
static cudaError_t absorb_dispatch(const mla_config& c, const void* qn, const void* qr,
                                   const int32_t* pos, const void* w, void* q, int n,
                                   cudaStream_t st) {
  if (c.kv_rank <= 256) return absorb_go<T, 1>(c, qn, qr, pos, w, q, n, st);
  if (c.kv_rank <= 512) return absorb_go<T, 2>(c, qn, qr, pos, w, q, n, st);
  return absorb_go<T, 4>(c, qn, qr, pos, w, q, n, st);
}

cudaError_t launch_absorb(const mla_config& c, const void* q_nope, const void* q_rope,
                          const int32_t* pos, const void* w_uk, void* q_out, int n,
                          cudaStream_t st) {
  if (c.dtype == MLA_BF16)
    return absorb_dispatch<__nv_bfloat16>(c, q_nope, q_rope, pos, w_uk, q_out, n, st);
  return absorb_dispatch<float>(c, q_nope, q_rope, pos, w_uk, q_out, n, st);
}

// ------------------------------------------------------------------------------------------
// Append: one warp per new row (append_row.cuh).
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
append_kernel(const T* __restrict__ ckv, const T* __restrict__ kr, const float* __restrict__ gamma,
              const int32_t* __restrict__ seq, const int32_t* __restrict__ pos,
              const int32_t* __restrict__ table, int batch, int max_blocks, T* __restrict__ pool,
              int num_blocks, int n, int r, int dr, int bs, float eps, float base,
              uint32_t* err, bool vec) {
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  wait_prior_grid();
  if (row >= n) return;
  append_row<T>(row, lane, ckv, kr, gamma, seq, pos, table, batch, max_blocks, pool, num_blocks,
                r, dr, bs, eps, base, err, vec);
}

cudaError_t launch_append(const mla_config& c, const void* ckv, const void* kr,
                          const float* gamma, const int32_t* seq, const int32_t* pos,
                          const int32_t* table, int batch, int max_blocks, void* pool,
                          int num_blocks, int n, uint32_t* err, cudaStream_t st) {
  const int threads = 256, rows_per_cta = threads / 32;
  const int grid = (n + rows_per_cta - 1) / rows_per_cta;
  if (c.dtype == MLA_BF16) {
    // contiguous 16-byte pieces per lane: r a multiple of 256 (at most 1024), aligned rows
    const bool vec = c.kv_rank % 256 == 0 && c.kv_rank <= 1024 && ((uintptr_t)ckv & 15) == 0 &&
                     ((uintptr_t)gamma & 15) == 0 && ((uintptr_t)pool & 15) == 0 &&
                     ((c.kv_rank + c.rope_dim) * 2) % 16 == 0;
    return launch_pdl(append_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, st,
                      (const __nv_bfloat16*)ckv, (const __nv_bfloat16*)kr, gamma, seq, pos, table,
                      batch, max_blocks, (__nv_bfloat16*)pool, num_blocks, n, c.kv_rank,
                      c.rope_dim, c.block_size, c.rms_eps, c.rope_base, err, vec);
  }
  return launch_pdl(append_kernel<float>, dim3(grid), dim3(threads), 0, st, (const float*)ckv,
                    (const float*)kr, gamma, seq, pos, table, batch, max_blocks, (float*)pool,
                    num_blocks, n, c.kv_rank, c.rope_dim, c.block_size, c.rms_eps, c.rope_base,
                    err, false);
}

// ------------------------------------------------------------------------------------------
// Output: o[n,h,i] = sum_j W_UV[h,i,j] * lat[n,h,j]. One CTA per (16 tokens, head); each warp
// streams whole rows of W_UV[h] (coalesced) against the 16 latent rows held in shared memory.
// ------------------------------------------------------------------------------------------
constexpr int kOutTokens = 16;

template <typename T>
__global__ void __launch_bounds__(256)
output_kernel(const float* __restrict__ lat, const T* __restrict__ w_uv, T* __restrict__ o, int n,
              int H, int dv, int r) {
  extern __shared__ float s_lat[];  // kOutTokens x r
  wait_prior_grid();
  const int h = blockIdx.y;
  const int n0 = blockIdx.x * kOutTokens;
  const int nt = min(kOutTokens, n - n0);
  for (int idx = threadIdx.x; idx < kOutTokens * r; idx += blockDim.x) {
    const int t = idx / r, j = idx - t * r;
    s_lat[idx] = t < nt ? lat[((size_t)(n0 + t) * H + h) * r + j] : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int i = warp; i < dv; i += nwarps) {
    const T* wrow = w_uv + ((size_t)h * dv + i) * r;
    float acc[kOutTokens];
#pragma unroll
    for (int t = 0; t < kOutTokens; ++t) acc[t] = 0.f;
    for (int j = lane; j < r; j += 32) {
      const float wv = to_f32(wrow[j]);
#pragma unroll
      for (int t = 0; t < kOutTokens; ++t) acc[t] = fmaf(wv, s_lat[t * r + j], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kOutTokens; ++t) {
      const float v = warp_sum(acc[t]);
      if (lane == 0 && t < nt) o[((size_t)(n0 + t) * H + h) * dv + i] = from_f32<T>(v);
    }
  }
}

cudaError_t launch_output(const mla_config& c, const float* lat, const void* w_uv, void* o,
                          int n, cudaStream_t st) {
  const size_t smem = sizeof(float) * kOutTokens * c.kv_rank;
  dim3 grid((n + kOutTokens - 1) / kOutTokens, c.num_heads);
  if (c.dtype == MLA_BF16) {
    auto k = output_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(k, grid, dim3(256), smem, st, lat, (const __nv_bfloat16*)w_uv,
                      (__nv_bfloat16*)o, n, c.num_heads, c.head_dim_v, c.kv_rank);
  } else {
    auto k = output_kernel<float>;
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(k, grid, dim3(256), smem, st, lat, (const float*)w_uv, (float*)o, n,
                      c.num_heads, c.head_dim_v, c.kv_rank);
  }
}

}  // namespace mla
