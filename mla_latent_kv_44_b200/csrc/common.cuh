// Internal declarations shared by the host API and the kernels of libmla.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "mla.h"

namespace mla {

// Work ranges the decode planner cuts every call into. 74 = one range per pair of SMs on a
// 148-SM B200 (the tensor-core kernel runs one CTA pair per range); the CUDA-core kernel
// uses the same schedule.
constexpr int kRanges = 74;
// Tokens per chunk of decode work (one tensor-core tile; one 64-token cache block).
constexpr int kChunk = 64;
// A split row range produces at most this many partial results per call.
constexpr int kMaxPartials = 2 * kRanges;

// A contiguous run of chunks of one (sequence, query token) row group.
struct Segment {
  int32_t bt;        // b * q_per_seq + t
  int32_t chunk_lo;  // first 64-row chunk
  int32_t chunk_hi;  // one past the last chunk
  int32_t slot;      // partial-result slot, or -1 when the segment covers the whole row group
};

// Byte offsets of the workspace regions (all 256-byte aligned).
struct WorkspaceLayout {
  size_t header;       // int32[64]: [0] segment count, [1] ranges used, [2] total chunks
  size_t range_begin;  // int32[kRanges + 1]: first segment of each range
  size_t segments;     // Segment[kRanges + BT]
  size_t bt_slot0;     // int32[BT]: first partial slot of a split row group (its slots are
                       // consecutive), -1 for a row group in one segment
  size_t bt_nseg;      // int32[BT]: number of segments of each row group (0: invalid length)
  size_t bt_len;       // int32[BT]: rows attended by each row group
  size_t bt_chunk0;    // int32[BT]: exclusive prefix of chunk counts
  size_t part_lse;     // float[kMaxPartials][H]
  size_t part_o;       // float[kMaxPartials][H][r]
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(int H, int r, int bt_count) {
  WorkspaceLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L.header = take(64 * sizeof(int32_t));
  L.range_begin = take((kRanges + 1) * sizeof(int32_t));
  L.segments = take(size_t(kRanges + bt_count) * sizeof(Segment));
  L.bt_slot0 = take(size_t(bt_count) * sizeof(int32_t));
  L.bt_nseg = take(size_t(bt_count) * sizeof(int32_t));
  L.bt_len = take(size_t(bt_count) * sizeof(int32_t));
  L.bt_chunk0 = take(size_t(bt_count) * sizeof(int32_t));
  L.part_lse = take(size_t(kMaxPartials) * H * sizeof(float));
  L.part_o = take(size_t(kMaxPartials) * H * r * sizeof(float));
  L.total = off;
  return L;
}

// Everything the decode stages need, resolved to device pointers.
struct DecodeParams {
  const void* q;
  const void* pool;
  const int32_t* table;
  const int32_t* seq_lens;
  float* out;
  float* lse;  // may be null
  uint32_t* err;
  // workspace regions
  int32_t* header;
  int32_t* range_begin;
  Segment* segments;
  int32_t* bt_slot0;
  int32_t* bt_nseg;
  int32_t* bt_len;
  int32_t* bt_chunk0;
  float* part_lse;
  float* part_o;
  const float* row_scale;  // fp8 cache: one fp32 scale per pool row (null otherwise)
  // shapes
  int32_t H, r, dr, D, bs, max_blocks, num_blocks, batch, T, BT;
  float scale;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// RoPE angle of pair i at position p, in double: p * base^(-2i/d_r).
__device__ __forceinline__ void rope_cos_sin(int p, int i, int dr, float base, double* c,
                                             double* s) {
  double theta = pow((double)base, -2.0 * (double)i / (double)dr);
  sincos((double)p * theta, s, c);
}

// Programmatic dependent launch: every kernel of the library is launched so that it may start
// while the previous kernel on the stream is still finishing, and waits here, after its own
// set-up and before it touches global memory, until that kernel has completed and its writes
// are visible. Launched without the attribute, the wait returns at once.
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- launchers (defined in the .cu files; return cudaGetLastError()) ----
cudaError_t launch_absorb(const mla_config& c, const void* q_nope, const void* q_rope,
                          const int32_t* pos, const void* w_uk, void* q_out, int n,
                          cudaStream_t st);
cudaError_t launch_append(const mla_config& c, const void* ckv, const void* kr,
                          const float* gamma, const int32_t* seq, const int32_t* pos,
                          const int32_t* table, int batch, int max_blocks, void* pool,
                          int num_blocks, int n, uint32_t* err, cudaStream_t st);
cudaError_t launch_plan(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_attend_simt(const mla_config& c, const DecodeParams& p, cudaStream_t st);
cudaError_t launch_attend_tc(const mla_config& c, const DecodeParams& p, cudaStream_t st);
bool tc_supported(const mla_config& c);
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t st);
// fp8 (e4m3) latent cache: rows of the pool are codes, p.row_scale their scales
cudaError_t launch_attend_simt_fp8(const mla_config& c, const DecodeParams& p, cudaStream_t st);
cudaError_t launch_append_fp8(const mla_config& c, const void* ckv, const void* kr,
                              const float* gamma, const int32_t* seq, const int32_t* pos,
                              const int32_t* table, int batch, int max_blocks, uint8_t* pool,
                              float* row_scale, int num_blocks, int n, uint32_t* err,
                              cudaStream_t st);
cudaError_t launch_output(const mla_config& c, const float* lat, const void* w_uv, void* o,
                          int n, cudaStream_t st);
bool absorb_tc_supported(const mla_config& c);
bool output_tc_supported(const mla_config& c);
cudaError_t launch_absorb_tc(const mla_config& c, const void* q_nope, const void* q_rope,
                             const int32_t* pos, const void* w_uk, void* q_out, int n,
                             uint32_t* err, cudaStream_t st);
cudaError_t launch_output_tc(const mla_config& c, const float* lat, const void* w_uv, void* o,
                             int n, uint32_t* err, cudaStream_t st);
// The fused step's first launch: absorb tiles, append rows and the planner as CTA roles of one
// grid (bf16, shapes where absorb_tc_supported and append's vector path hold).
cudaError_t launch_step_prep(const mla_config& c, const void* q_nope, const void* q_rope,
                             const int32_t* pos, const void* w_uk, void* q_out, int n,
                             const void* ckv, const void* kr, const float* gamma,
                             const int32_t* seq, const DecodeParams& p, void* pool,
                             cudaStream_t st);

}  // namespace mla
