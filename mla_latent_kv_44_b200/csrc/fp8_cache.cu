// FP8 latent cache ("MLA from scratch in PyTorch", What's not in this implementation: the
// latent cache can be quantised to FP8): the cache row of a new token, [RMSNorm(c_kv) * gamma
// ‖ RoPE(k_rope)] in fp32, stored as e4m3 codes with one fp32 scale per row,
//   scale = max_j |y_j| / 448 (1 for an all-zero row),  code_j = e4m3(y_j / scale),
// rounded to nearest even and saturated at the largest finite e4m3 value (448), so that a row
// reads back as code_j * scale. Half the bytes of a bf16 row (576 + 4 against 1152 at the
// DeepSeek-V2 shape). One warp per row, as the bf16 append. The decode either reads the codes
// on CUDA cores (decode_simt.cu) or, where the tensor-core attention applies, expands the
// step's blocks to bf16 in its workspace first (below) and runs that kernel over them: the
// expansion costs a read of the fp8 rows and a write of bf16 ones, so the fp8 cache saves
// memory, not time.
#include <cuda_fp8.h>

#include "common.cuh"

namespace mla {
namespace {

constexpr float kE4m3Max = 448.f;

template <typename T>
__global__ void __launch_bounds__(256)
append_fp8_kernel(const T* __restrict__ ckv, const T* __restrict__ kr,
                  const float* __restrict__ gamma, const int32_t* __restrict__ seq,
                  const int32_t* __restrict__ pos, const int32_t* __restrict__ table, int batch,
                  int max_blocks, uint8_t* __restrict__ pool, float* __restrict__ row_scale,
                  int num_blocks, int n, int r, int dr, int bs, float eps, float base,
                  uint32_t* err) {
  extern __shared__ float ybuf[];  // per warp: the row's r + dr values in fp32
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  wait_prior_grid();
  if (row >= n) return;
  const int b = seq[row], p = pos[row];
  if (b < 0 || b >= batch || p < 0 || (int64_t)p >= (int64_t)max_blocks * bs) {
    if (lane == 0) set_error(err, MLA_DEV_OOB_POS);
    return;
  }
  const int blk = table[(size_t)b * max_blocks + p / bs];
  if (blk < 0 || blk >= num_blocks) {
    if (lane == 0) set_error(err, MLA_DEV_OOB_BLOCK);
    return;
  }
  const int D = r + dr;
  float* y = ybuf + warp * D;
  const T* x = ckv + (size_t)row * r;
  float ss = 0.f;
  for (int j = lane; j < r; j += 32) {
    const float v = to_f32(x[j]);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / (float)r + eps);
  float amax = 0.f;
  for (int j = lane; j < r; j += 32) {
    y[j] = to_f32(x[j]) * inv * gamma[j];
    amax = fmaxf(amax, fabsf(y[j]));
  }
  const T* k = kr + (size_t)row * dr;
  for (int i = lane; i < dr / 2; i += 32) {
    double c, s;
    rope_cos_sin(p, i, dr, base, &c, &s);
    const double x0 = to_f32(k[2 * i]), x1 = to_f32(k[2 * i + 1]);
    y[r + 2 * i] = (float)(x0 * c - x1 * s);
    y[r + 2 * i + 1] = (float)(x0 * s + x1 * c);
    amax = fmaxf(amax, fmaxf(fabsf(y[r + 2 * i]), fabsf(y[r + 2 * i + 1])));
  }
  amax = warp_max(amax);
  __syncwarp();
  const float scale = amax > 0.f ? amax / kE4m3Max : 1.f;
  const size_t slot = (size_t)blk * bs + (p % bs);
  uint8_t* dst = pool + slot * (size_t)D;
  for (int j = lane; j < D; j += 32)
    dst[j] = (uint8_t)__nv_cvt_float_to_fp8(y[j] / scale, __NV_SATFINITE, __NV_E4M3);
  if (lane == 0) row_scale[slot] = scale;
}

// The step's fp8 rows back to bf16 for the tensor-core decode: block j of sequence b (if it
// holds rows of the sequence) into scratch block b * max_blocks + j, with the scratch table.
// Grid (max_blocks, batch); a thread per 4 codes. Out-of-pool ids are flagged and read as
// block 0.
__global__ void __launch_bounds__(256)
dequant_fp8_kernel(const uint8_t* __restrict__ pool, const float* __restrict__ row_scale,
                   const int32_t* __restrict__ table, const int32_t* __restrict__ seq_lens,
                   int max_blocks, int num_blocks, int bs, int D, __nv_bfloat16* __restrict__ out,
                   int32_t* __restrict__ out_table, uint32_t* err) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int dst_blk = b * max_blocks + j;
  wait_prior_grid();
  if (threadIdx.x == 0) out_table[(size_t)b * max_blocks + j] = dst_blk;
  const int len = seq_lens[b];
  if ((int64_t)j * bs >= (int64_t)len) return;
  int blk = table[(size_t)b * max_blocks + j];
  if (blk < 0 || blk >= num_blocks) {
    if (threadIdx.x == 0) set_error(err, MLA_DEV_OOB_BLOCK);
    blk = 0;
  }
  const uint32_t* src = (const uint32_t*)(pool + (size_t)blk * bs * D);
  uint2* dst = (uint2*)(out + (size_t)dst_blk * bs * D);
  const int quads = bs * D / 4;  // D is a multiple of 8
  for (int i = threadIdx.x; i < quads; i += blockDim.x) {
    const uint32_t u = src[i];
    const float sc = row_scale[(size_t)blk * bs + (4 * i) / D];
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)((u >> (8 * k)) & 0xffu),
                                                   __NV_E4M3);
      v[k] = __half2float(__half(h)) * sc;
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
    dst[i] = make_uint2(*(const uint32_t*)&lo, *(const uint32_t*)&hi);
  }
}

}  // namespace

cudaError_t launch_dequant_fp8(const uint8_t* pool, const float* row_scale, const int32_t* table,
                               const int32_t* seq_lens, int batch, int max_blocks, int num_blocks,
                               int bs, int D, void* out, int32_t* out_table, uint32_t* err,
                               cudaStream_t st) {
  return launch_pdl(dequant_fp8_kernel, dim3(max_blocks, batch), dim3(256), 0, st, pool,
                    row_scale, table, seq_lens, max_blocks, num_blocks, bs, D,
                    (__nv_bfloat16*)out, out_table, err);
}

cudaError_t launch_append_fp8(const mla_config& c, const void* ckv, const void* kr,
                              const float* gamma, const int32_t* seq, const int32_t* pos,
                              const int32_t* table, int batch, int max_blocks, uint8_t* pool,
                              float* row_scale, int num_blocks, int n, uint32_t* err,
                              cudaStream_t st) {
  const int warps = 8;
  const size_t smem = (size_t)warps * (c.kv_rank + c.rope_dim) * sizeof(float);
  const dim3 grid((n + warps - 1) / warps);
  if (c.dtype == MLA_BF16)
    return launch_pdl(append_fp8_kernel<__nv_bfloat16>, grid, dim3(32 * warps), smem, st,
                      (const __nv_bfloat16*)ckv, (const __nv_bfloat16*)kr, gamma, seq, pos, table,
                      batch, max_blocks, pool, row_scale, num_blocks, n, c.kv_rank, c.rope_dim,
                      c.block_size, c.rms_eps, c.rope_base, err);
  return launch_pdl(append_fp8_kernel<float>, grid, dim3(32 * warps), smem, st,
                    (const float*)ckv, (const float*)kr, gamma, seq, pos, table, batch,
                    max_blocks, pool, row_scale, num_blocks, n, c.kv_rank, c.rope_dim,
                    c.block_size, c.rms_eps, c.rope_base, err);
}

}  // namespace mla
