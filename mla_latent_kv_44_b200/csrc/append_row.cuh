// One row of mla_append_latent, done by one warp: RMSNorm of the new c_kv row (fp32
// statistics, lane-sequential partial sums, then a butterfly) times gamma, RoPE of the shared
// key (angle and rotation in double), both stored into the row's cache slot, bf16 rounded to
// nearest even. Shared by the append kernel (proj_kernels.cu) and the fused step kernel
// (proj_tc.cu).
#pragma once

#include "common.cuh"

namespace mla {

// vec: bf16 rows, r a multiple of 256 (at most 1024), 16-byte aligned -- lane l then owns the
// r/32 contiguous values [l * r/32, (l+1) * r/32), up to four 16-byte pieces loaded together.
template <typename T>
__device__ __forceinline__ void append_row(int row, int lane, const T* __restrict__ ckv,
                                           const T* __restrict__ kr,
                                           const float* __restrict__ gamma,
                                           const int32_t* __restrict__ seq,
                                           const int32_t* __restrict__ pos,
                                           const int32_t* __restrict__ table, int batch,
                                           int max_blocks, T* __restrict__ pool, int num_blocks,
                                           int r, int dr, int bs, float eps, float base,
                                           uint32_t* err, bool vec) {
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
  const T* x = ckv + (size_t)row * r;
  T* dst = pool + ((size_t)blk * bs + (p % bs)) * (size_t)(r + dr);
  if (vec) {
    // bf16 rows, r a multiple of 256, 16-byte aligned: lane l owns the r/32 contiguous values
    // [l * r/32, (l+1) * r/32), up to four 16-byte pieces loaded together
    const int E = r / 32, pieces = E / 8;
    uint4 xv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < pieces) xv[k] = ((const uint4*)(x + lane * E))[k];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= pieces) break;
      const uint32_t w[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float a0 = __uint_as_float(w[u] << 16), a1 = __uint_as_float(w[u] & 0xffff0000u);
        ss = fmaf(a0, a0, ss);
        ss = fmaf(a1, a1, ss);
      }
    }
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)r + eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= pieces) break;
      const float4 g0 = ((const float4*)(gamma + lane * E))[2 * k];
      const float4 g1 = ((const float4*)(gamma + lane * E))[2 * k + 1];
      const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const uint32_t w[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
      uint32_t o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float a0 = __uint_as_float(w[u] << 16), a1 = __uint_as_float(w[u] & 0xffff0000u);
        const __nv_bfloat162 v = __floats2bfloat162_rn(a0 * inv * gg[2 * u], a1 * inv * gg[2 * u + 1]);
        o[u] = *reinterpret_cast<const uint32_t*>(&v);
      }
      ((uint4*)(dst + lane * E))[k] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    float ss = 0.f;
    for (int j = lane; j < r; j += 32) {
      const float v = to_f32(x[j]);
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)r + eps);
    for (int j = lane; j < r; j += 32) dst[j] = from_f32<T>(to_f32(x[j]) * inv * gamma[j]);
  }
  const T* k = kr + (size_t)row * dr;
  for (int i = lane; i < dr / 2; i += 32) {
    double c, s;
    rope_cos_sin(p, i, dr, base, &c, &s);
    const double x0 = to_f32(k[2 * i]), x1 = to_f32(k[2 * i + 1]);
    dst[r + 2 * i] = from_f32<T>((float)(x0 * c - x1 * s));
    dst[r + 2 * i + 1] = from_f32<T>((float)(x0 * s + x1 * c));
  }
}

}  // namespace mla
