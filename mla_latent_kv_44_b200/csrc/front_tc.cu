// Decode front end: hidden states x -> the library's per-token inputs, for sm_100a.
//   q_nope    = W_UQ RMSNorm(W_DQ x) per head     ("MLA from scratch in PyTorch", The
//               (or W_Q x with a full-rank query)   MLAAttention module: c_q = norm(W_DQ x),
//                                                   q = W_UQ c_q)
//   q_rope    = W_QR x per head                   ("Multi-head latent attention",
//   ckv_raw   = W_DKV x                             _project_mla: the RoPE query and key are
//   krope_raw = W_KR x                              projected from x; one key row shared by
//                                                   all heads)
// Weights use the nn.Linear layout (out_features, in_features). At decode the tokens are few
// and the weights many (DeepSeek-V2: 156 MB of bf16 weights for 64 tokens), so every product
// is a weight stream: the weight rows are the MMA's M = 128 side, the tokens its N side, and
// the K dimension is split across CTAs so that the SMs get about equal shares. Each CTA
// streams its K range of one 128-row weight tile through a 4-stage TMA ring (128-byte swizzled
// 64-wide slabs of the weight and of the tokens), one thread issues the MMAs into fp32 TMEM,
// and the CTA writes its fp32 partial sums. A second kernel adds the K splits in a fixed order
// (deterministic) and writes the outputs, normalising the c_q rows (RMSNorm, fp32 statistics)
// on the way; a product left in one split with no norm is written by the first kernel alone. One launch of each covers all four projections from x (a table of up to four
// weight segments); the W_UQ product follows with its own pair. fp32 configurations take a
// CUDA-core kernel that writes the same partial layout (one split).
// Every mbarrier wait gives up after 1 s: the kernel then sets MLA_DEV_WAIT_TIMEOUT, waits
// (bounded) for what it issued, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_map.h"

namespace mla {
namespace {

constexpr unsigned long long kFrontTimeoutNs = 1000000000ull;
constexpr int kFrontRows = 128;      // weight rows per CTA = MMA M
constexpr int kFrontStages = 4;
constexpr int kFrontMaxTok = 128;    // tokens per CTA at most = MMA N = TMEM columns
constexpr int kFrontSlab = 64;       // bf16 values per 128-byte swizzled row
constexpr int kFrontMaxSegs = 4;
constexpr uint32_t kFrontTmemCols = 128;
constexpr int kMaxSplits = 8;        // K splits of one product at most

struct FrontSeg {
  float* part;    // partial sums (splits, n, rows) fp32
  void* out;      // with one split and no norm: the bf16 output (n, rows), written directly
  int rows;       // output features
  int tile0;      // first M tile of the segment in the grid
};

struct LinearArgs {
  FrontSeg seg[kFrontMaxSegs];
  const float* wf[kFrontMaxSegs];  // fp32 weights (CUDA-core kernel only)
  int nseg, n, K, ldx, splits, ntile;  // ldx: elements between consecutive rows of x
  uint32_t* err;
};

__device__ __forceinline__ bool front_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > kFrontTimeoutNs) {
      set_error(err, MLA_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ int front_segment(const LinearArgs& a, int tile) {
  int s = 0;
  while (s + 1 < a.nseg && tile >= a.seg[s + 1].tile0) ++s;
  return s;
}

// Grid (M tiles of all segments, K splits, token tiles); 128 threads. Shared memory: the ring
// of (weight slab: 128 rows x 128 B, token slab: ntile rows x 128 B) stages, then barriers.
__global__ void __launch_bounds__(128)
linear_tc_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                 const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tm3,
                 const __grid_constant__ CUtensorMap tmx, const LinearArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = front_segment(a, blockIdx.x);
  const FrontSeg sg = a.seg[s];
  const CUtensorMap* tw = s == 0 ? &tm0 : s == 1 ? &tm1 : s == 2 ? &tm2 : &tm3;
  const int row0 = (blockIdx.x - sg.tile0) * kFrontRows;
  const int slabs = (a.K + kFrontSlab - 1) / kFrontSlab;  // a ragged last slab reads zeros
  const int k0 = (int)((long long)blockIdx.y * slabs / a.splits);
  const int k1 = (int)((long long)(blockIdx.y + 1) * slabs / a.splits);
  const int nk = k1 - k0;
  const int t0 = blockIdx.z * a.ntile;
  const int ntok = min(a.ntile, a.n - t0);
  const int nmma = (ntok + 15) / 16 * 16;
  constexpr uint32_t kSlabA = kFrontRows * 128;                    // 16 KB
  const uint32_t slab_b = (uint32_t)((a.ntile * 128 + 1023) / 1024 * 1024);
  const uint32_t stage_bytes = kSlabA + slab_b;
  const uint32_t s0 = saddr(smem);
  uint8_t* ctl = smem + kFrontStages * stage_bytes;
  const uint32_t bar_full = saddr(ctl);                    // [stages]
  const uint32_t bar_empty = bar_full + 8 * kFrontStages;  // [stages]
  const uint32_t bar_done = bar_empty + 8 * kFrontStages;
  uint32_t* tmem_slot = (uint32_t*)(ctl + 16 * kFrontStages + 8);
  int* issued = (int*)(ctl + 16 * kFrontStages + 12);      // stages loaded, for the abort drain
  if (threadIdx.x == 0) {
    for (int i = 0; i < kFrontStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_done, 1);
    *issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(kFrontTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  wait_prior_grid();  // x (or c_q) comes from an earlier kernel

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      for (int j = 0; j < nk && ok; ++j) {
        const int st = j % kFrontStages;
        if (j >= kFrontStages)
          ok = front_wait(bar_empty + 8 * st, ((j / kFrontStages) - 1) & 1, a.err);
        if (!ok) break;
        const uint32_t sa = s0 + st * stage_bytes;
        mbar_expect_tx(bar_full + 8 * st, kSlabA + (uint32_t)a.ntile * 128);
        tma_load(sa, tw, bar_full + 8 * st, (k0 + j) * kFrontSlab, row0);
        tma_load(sa + kSlabA, &tmx, bar_full + 8 * st, (k0 + j) * kFrontSlab, t0);
        *issued = j + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc(kFrontRows, nmma, 0, 0);
      int j = 0;
      for (; j < nk && ok; ++j) {
        const int st = j % kFrontStages;
        ok = front_wait(bar_full + 8 * st, (j / kFrontStages) & 1, a.err);
        if (!ok) break;
        tc_after();
        const uint32_t sa = s0 + st * stage_bytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // 16 K values per MMA, 32 bytes into the swizzled rows
          mma_ss(tmem, sdesc(sa + 32 * ks, 16, 1024, 2), sdesc(sa + kSlabA + 32 * ks, 16, 1024, 2),
                 id, (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(bar_empty + 8 * st);
      }
      tc_commit(bar_done);  // every MMA issued above (none if the loop stopped at once)
    }
  }
  __syncwarp();
  ok = __syncthreads_and(ok);
  // all MMAs done; then TMEM lane i (weight row row0 + i), column t (token t0 + t)
  if (ok) ok = __syncthreads_and(front_wait(bar_done, 0, a.err));
  if (ok && nk > 0) {
    tc_after();
    const int row = row0 + 32 * warp + lane;
    float* part = sg.part + ((size_t)blockIdx.y * a.n + t0) * sg.rows + row;
    __nv_bfloat16* out = sg.out ? (__nv_bfloat16*)sg.out + (size_t)t0 * sg.rows + row : nullptr;
    for (int c0 = 0; c0 < nmma; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + c0, v);
      if (row < sg.rows) {
        if (out) {
#pragma unroll
          for (int cc = 0; cc < 32; ++cc)
            if (c0 + cc < ntok)
              out[(size_t)(c0 + cc) * sg.rows] = __float2bfloat16_rn(__uint_as_float(v[cc]));
        } else {
#pragma unroll
          for (int cc = 0; cc < 32; ++cc)
            if (c0 + cc < ntok) part[(size_t)(c0 + cc) * sg.rows] = __uint_as_float(v[cc]);
        }
      }
    }
  }
  tc_before();
  __syncthreads();
  tc_after();
  if (!ok && threadIdx.x == 0) {
    // copies that may still land, then the MMAs already committed
    const int loaded = *issued;
    for (int j = max(0, loaded - kFrontStages); j < loaded; ++j) {
      const uint64_t t_0 = globaltimer();
      while (!mbar_try(bar_full + 8 * (j % kFrontStages), (j / kFrontStages) & 1) &&
             globaltimer() - t_0 < kFrontTimeoutNs) {
      }
    }
    const uint64_t t_0 = globaltimer();
    while (!mbar_try(bar_done, 0) && globaltimer() - t_0 < kFrontTimeoutNs) {
    }
  }
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kFrontTmemCols)
                 : "memory");
}

// CUDA-core version of the same partial sums for fp32 (one split): thread (row, token) takes
// one dot product; a CTA shares a token's x row in shared memory for 128 weight rows.
__global__ void __launch_bounds__(128)
linear_simt_kernel(const float* x, const LinearArgs a) {
  extern __shared__ float xs[];  // one token's K values
  const int s = front_segment(a, blockIdx.x);
  const FrontSeg sg = a.seg[s];
  const int row = (blockIdx.x - sg.tile0) * kFrontRows + threadIdx.x;
  wait_prior_grid();
  for (int t = blockIdx.z; t < a.n; t += gridDim.z) {
    __syncthreads();
    for (int k = threadIdx.x; k < a.K; k += blockDim.x) xs[k] = x[(size_t)t * a.ldx + k];
    __syncthreads();
    if (row < sg.rows) {
      const float* wr = a.wf[s] + (size_t)row * a.K;
      float acc = 0.f;
      for (int k = 0; k < a.K; ++k) acc = fmaf(wr[k], xs[k], acc);
      sg.part[(size_t)t * sg.rows + row] = acc;
    }
  }
}

// Sum of the K splits in split order and the outputs in the config's dtype. A 1-D grid over
// the (token, segment, 1024-column block) triples that exist, in that order; a normalised
// segment (c_q) is one block per token, since its statistics need the whole row:
// y = (x * gamma) / sqrt(mean(x^2) + eps), in fp32 (gamma is read with the partial sums).
struct ReduceArgs {
  const float* part[kFrontMaxSegs];
  void* out[kFrontMaxSegs];
  int rows[kFrontMaxSegs];
  int blocks[kFrontMaxSegs];  // blocks of each segment per token
  int per_token;              // sum of blocks
  int n, splits, norm_seg;
  const float* gamma;
  float eps;
};

constexpr int kReduceCols = 1024;  // columns per block of a segment that is not normalised
constexpr int kReduceThreads = 256;
constexpr int kReduceVec = kReduceCols / kReduceThreads;

template <typename T>
__global__ void __launch_bounds__(kReduceThreads) front_reduce_kernel(const ReduceArgs a) {
  extern __shared__ float rowbuf[];  // the normalised segment's row
  __shared__ float red[kReduceThreads / 32];
  const int t = blockIdx.x / a.per_token;
  int b = blockIdx.x - t * a.per_token, s = 0;
  while (b >= a.blocks[s]) b -= a.blocks[s++];
  const int rows = a.rows[s];
  const bool norm = (s == a.norm_seg);
  const int c_lo = norm ? 0 : b * kReduceCols;
  const int c_hi = norm ? rows : min(rows, c_lo + kReduceCols);
  const float* p = a.part[s] + (size_t)t * rows;
  T* out = (T*)a.out[s] + (size_t)t * rows;
  const size_t plane = (size_t)a.n * rows;
  wait_prior_grid();
  float ss = 0.f;
  for (int c0 = c_lo; c0 < c_hi; c0 += kReduceCols) {
    // every split's value of kReduceVec columns in flight at once, then added in split order
    float v[kReduceVec][kMaxSplits];
    float g[kReduceVec];
#pragma unroll
    for (int u = 0; u < kReduceVec; ++u) {
      const int c = c0 + threadIdx.x + u * kReduceThreads;
#pragma unroll
      for (int k = 0; k < kMaxSplits; ++k)
        v[u][k] = (k < a.splits && c < c_hi) ? p[k * plane + c] : 0.f;
      g[u] = (norm && c < c_hi) ? a.gamma[c] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kReduceVec; ++u) {
      const int c = c0 + threadIdx.x + u * kReduceThreads;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxSplits; ++k)
        if (k < a.splits) acc += v[u][k];
      if (c < c_hi) {
        if (norm) {
          rowbuf[c] = acc * g[u];
          ss = fmaf(acc, acc, ss);
        } else {
          out[c] = from_f32<T>(acc);
        }
      }
    }
  }
  if (!norm) return;
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < kReduceThreads / 32; ++w) tot += red[w];
  const float inv = rsqrtf(tot / (float)rows + a.eps);
  for (int c = threadIdx.x; c < rows; c += kReduceThreads)
    out[c] = from_f32<T>(rowbuf[c] * inv);
}

int front_ntile(int n) { return std::min(kFrontMaxTok, (n + 15) / 16 * 16); }

// K splits: the count (at most kMaxSplits, at least two slabs per split) with the fewest bytes
// per SM: its CTAs (rounded up to whole rounds over the 148 SMs) times the weight slabs of
// each, plus its share of the fp32 partial sums written and read back (none with one split
// and no norm, which the first kernel writes out directly).
int front_splits(int mtiles, int ttiles, int K, int n, int rows_total, bool norm) {
  const int slabs = (K + kFrontSlab - 1) / kFrontSlab;
  const int cap = std::max(1, std::min(kMaxSplits, slabs / 2));
  int best = 1;
  double best_cost = -1.0;
  for (int sp = 1; sp <= cap; ++sp) {
    const long long ctas = (long long)mtiles * ttiles * sp;
    const double weights = (double)((ctas + 147) / 148) * ((slabs + sp - 1) / sp) * 16384.0;
    const double parts = (sp == 1 && !norm) ? 0.0 : 8.0 * sp * n * (double)rows_total / 148.0;
    const double cost = weights + parts;
    if (best_cost < 0 || cost < best_cost) {
      best = sp;
      best_cost = cost;
    }
  }
  return best;
}

size_t front_smem(int ntile) {
  const size_t stage = (size_t)kFrontRows * 128 + (size_t)((ntile * 128 + 1023) / 1024 * 1024);
  return 1024 + kFrontStages * stage + 16 * kFrontStages + 64;
}

}  // namespace

// bf16 rows of K values whose byte length TMA can stride over (a multiple of 16 bytes); the
// last 64-wide slab may reach past K, where TMA fills zeros.
bool front_tc_supported(const mla_config& c, int K) {
  return c.dtype == MLA_BF16 && K % 8 == 0;
}

// Partial-sum buffer of one product: splits x n x rows fp32 (256-byte aligned sizes).
size_t front_part_bytes(const mla_config& c, int K, int n, const int* rows, int nseg,
                        bool norm) {
  int mt = 0, total = 0;
  for (int i = 0; i < nseg; ++i) {
    mt += (rows[i] + kFrontRows - 1) / kFrontRows;
    total += rows[i];
  }
  const int nt = (n + kFrontMaxTok - 1) / kFrontMaxTok;
  const int splits = front_tc_supported(c, K) ? front_splits(mt, nt, K, n, total, norm) : 1;
  return (size_t)splits * n * total * 4 + 256 * (size_t)nseg;
}

// y_s = W_s x for up to four weights W_s (rows[s] x K, nn.Linear layout) sharing the input
// x (n rows of K values, ldx elements apart); outputs in the config's dtype at out[s]
// (n x rows[s]); segment norm_seg (or -1) is RMS-normalised with gain gamma. `part` holds
// front_part_bytes(...).
cudaError_t launch_front_linear(const mla_config& c, const void* x, int n, int K, int ldx,
                                const void* const* w, const int* rows, void* const* out, int nseg,
                                int norm_seg, const float* gamma, float eps, void* part,
                                uint32_t* err, cudaStream_t st) {
  LinearArgs a{};
  ReduceArgs r{};
  int mt = 0, total = 0;
  char* pp = (char*)part;
  for (int i = 0; i < nseg; ++i) {
    a.seg[i].rows = rows[i];
    a.seg[i].tile0 = mt;
    mt += (rows[i] + kFrontRows - 1) / kFrontRows;
    total += rows[i];
  }
  const bool tc = front_tc_supported(c, K);
  const int ntile = front_ntile(n);
  const int nt = (n + ntile - 1) / ntile;
  const int splits =
      tc ? front_splits(mt, (n + kFrontMaxTok - 1) / kFrontMaxTok, K, n, total, norm_seg >= 0)
         : 1;
  // one split and no norm: the tensor-core kernel writes the bf16 outputs itself
  const bool direct = tc && splits == 1 && norm_seg < 0;
  for (int i = 0; i < nseg; ++i) {
    a.seg[i].part = (float*)pp;
    a.seg[i].out = direct ? out[i] : nullptr;
    r.part[i] = (const float*)pp;
    r.out[i] = out[i];
    r.rows[i] = rows[i];
    pp += ((size_t)splits * n * rows[i] * 4 + 255) / 256 * 256;
  }
  a.nseg = nseg;
  a.n = n;
  a.K = K;
  a.ldx = ldx;
  a.splits = splits;
  a.ntile = ntile;
  a.err = err;
  cudaError_t e;
  if (tc) {
    CUtensorMap tm[kFrontMaxSegs], tx;
    for (int i = 0; i < kFrontMaxSegs; ++i) {
      const int j = i < nseg ? i : 0;
      if (!make_bf16_map(&tm[i], w[j], (uint64_t)K, (uint64_t)rows[j], (uint64_t)K * 2,
                         kFrontRows))
        return cudaErrorInvalidValue;
    }
    if (!make_bf16_map(&tx, x, (uint64_t)K, (uint64_t)n, (uint64_t)ldx * 2, (uint32_t)ntile))
      return cudaErrorInvalidValue;
    const size_t smem = front_smem(ntile);
    e = cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(linear_tc_kernel, dim3(mt, splits, nt), dim3(128), smem, st, tm[0], tm[1],
                   tm[2], tm[3], tx, a);
  } else {
    for (int i = 0; i < nseg; ++i) a.wf[i] = (const float*)w[i];
    const size_t smem = (size_t)K * 4;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(linear_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(linear_simt_kernel, dim3(mt, 1, std::min(n, 64)), dim3(128), smem, st,
                   (const float*)x, a);
  }
  if (e != cudaSuccess || direct) return e;
  r.n = n;
  r.splits = splits;
  r.norm_seg = norm_seg;
  r.gamma = gamma;
  r.eps = eps;
  const size_t rsmem = norm_seg >= 0 ? (size_t)rows[norm_seg] * 4 : 0;
  if (rsmem > 48 * 1024) return cudaErrorInvalidValue;
  auto rk = c.dtype == MLA_BF16 ? front_reduce_kernel<__nv_bfloat16> : front_reduce_kernel<float>;
  r.per_token = 0;
  for (int i = 0; i < nseg; ++i) {
    r.blocks[i] = i == norm_seg ? 1 : (rows[i] + kReduceCols - 1) / kReduceCols;
    r.per_token += r.blocks[i];
  }
  return launch_pdl(rk, dim3((unsigned)n * r.per_token), dim3(kReduceThreads), rsmem, st, r);
}

}  // namespace mla
