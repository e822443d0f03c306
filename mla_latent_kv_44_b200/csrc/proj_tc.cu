// tcgen05 tensor-core projections of the bf16 decode step, for sm_100a:
//   absorbed query   Q[n, h, 0:r] = W_UK[h]^T q_nope[n, h]        ("DeepSeek MLA, Built From the
//                    Paper", 3 Matrix absorption: W_UK folds into the query)
//   output           o[n, h, :]   = W_UV[h] o_lat[n, h, :]         ("MLA from scratch in
//                    PyTorch", Absorbing projections: W_UV after the weighted sum)
// Per head both are small dense GEMMs whose cost is reading the weights once (16.8 MB each at
// H = 128, d = 128, r = 512). The weight tile is the M = 128 side of the MMA (latent dims for
// the query, output dims for the output), the tokens are its N side, so one CTA handles one
// (head, 128-row weight tile, token tile): TMA brings the weight tile and the bf16 query rows
// into shared memory in the 128-byte swizzled layout, one thread issues the MMAs into an fp32
// TMEM accumulator, and four warps read it back and store bf16. The output's latent operand is
// fp32 in memory; threads split it into two bf16 terms while writing it into the same
// swizzled layout, so the MMA's operands are bf16, its sums fp32, and the latent keeps about
// 16 significant bits.
// Every mbarrier wait gives up after 1 s: it then sets MLA_DEV_WAIT_TIMEOUT, waits (also
// bounded) for the copies and MMAs already issued, frees TMEM and returns without storing.
#include <algorithm>

#include "append_row.cuh"
#include "common.cuh"
#include "plan_body.cuh"
#include "tc_ptx.cuh"
#include "tma_map.h"

namespace mla {
namespace {

constexpr unsigned long long kProjTimeoutNs = 1000000000ull;
constexpr int kWRows = 128;        // weight rows per CTA = MMA M
constexpr int kMaxTokTile = 128;   // tokens per CTA at most = MMA N (TMEM columns)
constexpr uint32_t kProjTmemCols = 128;
constexpr int kSlab = 64;          // bf16 elements per 128-byte swizzled row
constexpr int kOutTokTile = 128;   // tokens per CTA of the output kernel at most
constexpr int kRopeVec = 8;        // 16-byte pieces of q_rope a thread has in flight
constexpr int kOutItems = kOutTokTile * 16 / 256;  // 8-float groups per thread and chunk

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint32_t* err) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > kProjTimeoutNs) {
      set_error(err, MLA_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Teardown after a failed wait: give a phase that may still complete its last chance.
__device__ void drain_bounded(uint32_t bar, uint32_t parity, uint32_t* err) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity))
    if (globaltimer() - t0 > kProjTimeoutNs) {
      set_error(err, MLA_DEV_WAIT_TIMEOUT);
      return;
    }
}

__device__ __forceinline__ uint32_t tmem_alloc_cols(uint32_t slot_addr) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
               "r"(kProjTmemCols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  return 0;
}
__device__ __forceinline__ void tmem_free_cols(uint32_t tmem) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
               "r"(kProjTmemCols)
               : "memory");
}

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

// ------------------------------------------------------------------------------------------
// Absorbed query. Grid (token tiles, ceil(r / 128), H); 128 threads.
// Shared memory: A = W_UK[h][:, j0 : j0+128] as two MN-major slabs (64 latent dims x d_h rows
// of 128 B each); B = q_nope[n0 : n0+tile, h, :] as d_h / 64 K-major slabs (tile rows x 128 B).
// D[j, n] = sum_i A[j, i] B[i, n] lands in TMEM lane j, column n.
// ------------------------------------------------------------------------------------------
struct AbsorbArgs {
  const __nv_bfloat16* q_rope;
  const int32_t* pos;
  __nv_bfloat16* q_out;
  uint32_t* err;
  int n, H, dh, r, dr, tile;
  float base;
};

// One CTA's work: token tile bx, latent tile jt, head h of a grid of (.., ny, nz) tiles.
__device__ __forceinline__ void absorb_tile(const CUtensorMap* tm_w, const CUtensorMap* tm_q,
                                            const AbsorbArgs& a, int bx, int jt, int h, int ny,
                                            int nz, uint8_t* smem_raw) {
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = bx * a.tile;
  const int ntok = min(a.tile, a.n - n0);
  const int nmma = round_up(ntok, 16);
  const int ksl = a.dh / kSlab;                      // K slabs of the query rows
  const uint32_t slab_a = (uint32_t)a.dh * 128;      // one 64-dim slab of the weight tile
  const uint32_t slab_b = (uint32_t)round_up(a.tile * 128, 1024);
  const uint32_t sA = saddr(smem);
  const uint32_t sB = sA + 2 * slab_a;
  uint8_t* ctl = smem + 2 * slab_a + ksl * slab_b;
  const uint32_t bar_full = saddr(ctl), bar_done = bar_full + 8;
  uint32_t* tmem_slot = (uint32_t*)(ctl + 16);
  int* flags = (int*)(ctl + 32);  // [0] MMAs issued
  const int j0 = jt * kWRows;
  const int halves = (j0 + kSlab < a.r) ? 2 : 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
    flags[0] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_cols(saddr(tmem_slot));
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  wait_prior_grid();

  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar_full, halves * slab_a + ksl * (uint32_t)a.tile * 128);
    for (int hf = 0; hf < halves; ++hf)
      tma_load(sA + hf * slab_a, tm_w, bar_full, j0 + kSlab * hf, h * a.dh);
    for (int k = 0; k < ksl; ++k)
      tma_load(sB + k * slab_b, tm_q, bar_full, h * a.dh + kSlab * k, n0);
  }

  // RoPE part of the query, while the copies are in flight: pairs (2i, 2i+1) rotated by
  // pos * base^(-2i/d_r), angle and rotation in double. The angles depend on the token only, so
  // each token of this tile is given to one CTA of the tile (CTA (jt, h) takes the tokens
  // t = jt + ny * h, ...), which takes the d_r/2 sin/cos pairs once into shared memory
  // and rotates the token's query in every head.
  const int D = a.r + a.dr;
  const int half = a.dr / 2;
  double* cs_tab = (double*)(ctl + 64);  // [2][half] cos, sin
  for (int t = jt + ny * h; t < ntok; t += ny * nz) {
    const int n = n0 + t;
    __syncthreads();  // the previous token's table is no longer read
    for (int i = threadIdx.x; i < half; i += blockDim.x)
      rope_cos_sin(a.pos[n], i, a.dr, a.base, &cs_tab[i], &cs_tab[half + i]);
    __syncthreads();
    // the token's q_rope rows of all heads (H x d_r bf16, contiguous) in 16-byte pieces, kRopeVec
    // pieces per thread loaded together, rotated, stored into the RoPE part of each Q row
    const int pieces = a.H * a.dr / 8;
    const uint4* src = (const uint4*)(a.q_rope + (size_t)n * a.H * a.dr);
    for (int base = 0; base < pieces; base += kRopeVec * blockDim.x) {
      uint4 x[kRopeVec];
#pragma unroll
      for (int k = 0; k < kRopeVec; ++k) {
        const int pc = base + k * blockDim.x + threadIdx.x;
        if (pc < pieces) x[k] = src[pc];
      }
#pragma unroll
      for (int k = 0; k < kRopeVec; ++k) {
        const int pc = base + k * blockDim.x + threadIdx.x;
        if (pc >= pieces) break;
        const int hh = pc / (a.dr / 8), e0 = (pc - hh * (a.dr / 8)) * 8;  // first of 8 values
        const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = e0 / 2 + u;  // pair index
          const double cs = cs_tab[i], sn = cs_tab[half + i];
          const double x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xffff0000u);
          o[u] = pack_bf16((float)(x0 * cs - x1 * sn), (float)(x0 * sn + x1 * cs));
        }
        *(uint4*)(a.q_out + ((size_t)n * a.H + hh) * D + a.r + e0) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }

  if (threadIdx.x == 0) {
    ok = wait_bounded(bar_full, 0, a.err);
    if (ok) {
      tc_after();
      const uint32_t id = idesc(kWRows, nmma, 0, 1);
      for (int ks = 0; ks < a.dh / 16; ++ks) {
        // A (MN-major): 16 K-rows further per step; LBO = distance of the two 64-dim slabs
        const uint64_t ad = sdesc(sA + ks * 2048, slab_a, 1024, 2);
        // B (K-major): 32 bytes further per step inside a slab, next slab every 4 steps
        const uint64_t bd = sdesc(sB + (ks >> 2) * slab_b + (ks & 3) * 32, 16, 1024, 2);
        mma_ss(tmem, ad, bd, id, ks > 0 ? 1u : 0u);
      }
      tc_commit(bar_done);
      flags[0] = 1;
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) ok = __syncthreads_and(wait_bounded(bar_done, 0, a.err));

  if (ok) {
    tc_after();
    const int j = j0 + 32 * warp + lane;
    for (int c0 = 0; c0 < nmma; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + c0, v);
      if (j < a.r) {
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int t = c0 + cc;
          if (t < ntok)
            a.q_out[((size_t)(n0 + t) * a.H + h) * D + j] = __float2bfloat16_rn(__uint_as_float(v[cc]));
        }
      }
    }
  }

  tc_before();
  __syncthreads();
  tc_after();
  if (!ok) {  // give in-flight copies and MMAs their chance to finish before freeing anything
    if (threadIdx.x == 0) drain_bounded(bar_full, 0, a.err);
    if (threadIdx.x == 32 && flags[0]) drain_bounded(bar_done, 0, a.err);
    __syncthreads();
  }
  if (warp == 1) tmem_free_cols(tmem);
}

__global__ void __launch_bounds__(128)
absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                 const AbsorbArgs a) {
  extern __shared__ uint8_t smem_raw[];
  absorb_tile(&tm_w, &tm_q, a, blockIdx.x, blockIdx.y, blockIdx.z, gridDim.y, gridDim.z, smem_raw);
}

// ------------------------------------------------------------------------------------------
// The fused step's first launch. Absorbing the query, appending the new cache rows and
// planning the decode do not depend on one another, so they run as CTA roles of one grid
// instead of three launches that wait for each other: CTA 0 runs the planner (the longest
// serial job, so it starts first), CTAs 1 .. app_ctas append four rows each (one warp per
// row), and the rest are the absorbed query's tiles. Each role waits for the previous grid
// on the stream before it touches global memory.
// ------------------------------------------------------------------------------------------
constexpr int kPrepThreads = 128;

struct PrepArgs {
  AbsorbArgs ab;             // absorb (n tokens; pos and base shared with the append)
  int ax, ay, az;            // the absorb tiles: token tiles x latent tiles x heads
  const __nv_bfloat16* ckv;  // append: raw rows (n, r) and (n, d_r), gain, sequence of each
  const __nv_bfloat16* kr;
  const float* gamma;
  const int32_t* seq;
  __nv_bfloat16* pool;
  int app_ctas;
  float eps;
  bool vec;
  DecodeParams p;            // the planner's, and the cache shape for the append
};

__global__ void __launch_bounds__(kPrepThreads)
step_prep_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                 const PrepArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_a[32], s_b[32], s_carry[2];
  int id = (int)blockIdx.x;
  if (id == 0) {
    plan_body<kPrepThreads>(a.p, s_a, s_b, s_carry);
    return;
  }
  id -= 1;
  if (id < a.app_ctas) {
    const int row = id * (kPrepThreads / 32) + (int)(threadIdx.x >> 5);
    wait_prior_grid();
    if (row < a.ab.n)
      append_row<__nv_bfloat16>(row, threadIdx.x & 31, a.ckv, a.kr, a.gamma, a.seq, a.ab.pos,
                                a.p.table, a.p.batch, a.p.max_blocks, a.pool, a.p.num_blocks,
                                a.p.r, a.p.dr, a.p.bs, a.eps, a.ab.base, a.p.err, a.vec);
    return;
  }
  id -= a.app_ctas;
  const int x = id % a.ax, y = (id / a.ax) % a.ay, z = id / (a.ax * a.ay);
  absorb_tile(&tm_w, &tm_q, a.ab, x, y, z, a.ay, a.az, smem_raw);
}

// ------------------------------------------------------------------------------------------
// Output. Grid (token tiles, ceil(d_v / 128), H); 256 threads. The K = r contraction runs in
// chunks of 128 latent dims through two shared-memory stages: TMA brings W_UV[h][i0:i0+128,
// chunk] (K-major slabs of 128 rows x 128 B) while all threads write the chunk of o_lat as
// bf16 K-major slabs (tile rows x 128 B, 16-byte groups XOR-swizzled by row % 8). The fp32
// latent is split into two bf16 terms, hi = bf16(x) and lo = bf16(x - hi), and both are
// multiplied by the (exactly bf16) weights, so the product sees x to about 16 significant
// bits instead of bf16's 8.
// D[i, n] = sum_j W[i, j] lat[n, j] lands in TMEM lane i, column n.
// ------------------------------------------------------------------------------------------
struct OutputArgs {
  const float* lat;
  __nv_bfloat16* o;
  uint32_t* err;
  int n, H, dv, r, tile;
};

__global__ void __launch_bounds__(256)
output_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const OutputArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.y, h = blockIdx.z, n0 = blockIdx.x * a.tile;
  const int ntok = min(a.tile, a.n - n0);
  const int nmma = round_up(ntok, 16);
  const int i0 = mt * kWRows;
  constexpr uint32_t kSlabA = kWRows * 128;             // 16 KB
  const uint32_t slab_b = (uint32_t)round_up(a.tile * 128, 1024);
  const uint32_t stage_bytes = 2 * kSlabA + 4 * slab_b;  // W slabs, then hi and lo slabs
  const uint32_t s0 = saddr(smem);
  uint8_t* ctl = smem + 2 * stage_bytes;
  const uint32_t bar_full = saddr(ctl);   // [2]
  const uint32_t bar_done = bar_full + 16;  // [2]
  uint32_t* tmem_slot = (uint32_t*)(ctl + 32);
  int* flags = (int*)(ctl + 48);          // [0] chunks whose MMAs were committed, [1] loaded
  const int nchunks = (a.r + 127) / 128;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_done + 8 * s, 1);
    }
    flags[0] = 0;
    flags[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_cols(saddr(tmem_slot));
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  // The weights of chunk c go by TMA into stage c & 1 as soon as that stage is free (chunks 0
  // and 1 at once, before anything else reads memory). The latent of chunk c + 1 is loaded into
  // registers while chunk c's MMAs run: each thread holds kOutItems groups of 8 floats
  // (tile <= 64 tokens x 16 groups).
  auto issue_w = [&](int c) {
    const int s = c & 1;
    const int k0 = c * 128, nsl = min(128, a.r - k0) / kSlab;
    mbar_expect_tx(bar_full + 8 * s, nsl * kSlabA);
    for (int k = 0; k < nsl; ++k)
      tma_load(s0 + s * stage_bytes + k * kSlabA, &tm_w, bar_full + 8 * s, k0 + kSlab * k,
               h * a.dv + i0);
    flags[1] = c + 1;
  };
  wait_prior_grid();
  if (threadIdx.x == 0) {
    issue_w(0);
    if (nchunks > 1) issue_w(1);
  }
  float4 pf[2 * kOutItems];
  auto load_lat = [&](int c) {
    const int k0 = c * 128, groups = min(128, a.r - k0) / 8;
#pragma unroll
    for (int it = 0; it < kOutItems; ++it) {
      const int idx = threadIdx.x + it * blockDim.x;
      const int t = idx / groups, q = idx - t * groups;
      pf[2 * it] = pf[2 * it + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < ntok) {
        const float4* src =
            (const float4*)(a.lat + ((size_t)(n0 + t) * a.H + h) * a.r + k0 + 8 * q);
        pf[2 * it] = __ldg(src);
        pf[2 * it + 1] = __ldg(src + 1);
      }
    }
  };
  load_lat(0);

  bool ok = true;
  for (int c = 0; c < nchunks && ok; ++c) {
    const int s = c & 1;
    const uint32_t sA = s0 + s * stage_bytes, sB = sA + 2 * kSlabA;
    uint8_t* pB = smem + s * stage_bytes + 2 * kSlabA;
    const int k0 = c * 128;
    const int width = min(128, a.r - k0);   // 64 or 128 (r is a multiple of 64)
    if (c >= 2) {  // stage s is free once the MMAs of chunk c - 2 are done
      ok = __syncthreads_and(wait_bounded(bar_done + 8 * s, ((c - 2) >> 1) & 1, a.err));
      if (!ok) break;
      if (threadIdx.x == 0) issue_w(c);
    }
    // o_lat chunk -> hi and lo bf16 terms, swizzled K-major: row t, 16-byte group g of slab
    // k at g ^ (t & 7); the lo slabs follow the two hi slabs
    const int groups = width / 8;
#pragma unroll
    for (int it = 0; it < kOutItems; ++it) {
      const int idx = threadIdx.x + it * blockDim.x;
      const int t = idx / groups, q = idx - t * groups;
      if (t < a.tile) {
        const int k = q >> 3, g = q & 7;
        const float x[8] = {pf[2 * it].x, pf[2 * it].y, pf[2 * it].z, pf[2 * it].w,
                            pf[2 * it + 1].x, pf[2 * it + 1].y, pf[2 * it + 1].z, pf[2 * it + 1].w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * e]), h1 = __float2bfloat16_rn(x[2 * e + 1]);
          hi[e] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
          lo[e] = pack_bf16(x[2 * e] - __bfloat162float(h0), x[2 * e + 1] - __bfloat162float(h1));
        }
        const uint32_t off = k * slab_b + t * 128 + ((g ^ (t & 7)) << 4);
        *(uint4*)(pB + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *(uint4*)(pB + 2 * slab_b + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    if (c + 1 < nchunks) load_lat(c + 1);  // in flight during this chunk's MMAs
    fence_proxy_async();
    __syncthreads();
    if (threadIdx.x == 0) {
      ok = wait_bounded(bar_full + 8 * s, (c >> 1) & 1, a.err);
      if (ok) {
        tc_after();
        const uint32_t id = idesc(kWRows, nmma, 0, 0);
        for (int ks = 0; ks < width / 16; ++ks) {
          const uint64_t ad = sdesc(sA + (ks >> 2) * kSlabA + (ks & 3) * 32, 16, 1024, 2);
          const uint32_t b_off = (ks >> 2) * slab_b + (ks & 3) * 32;
          mma_ss(tmem, ad, sdesc(sB + b_off, 16, 1024, 2), id, (c > 0 || ks > 0) ? 1u : 0u);
          mma_ss(tmem, ad, sdesc(sB + 2 * slab_b + b_off, 16, 1024, 2), id, 1u);
        }
        tc_commit(bar_done + 8 * s);
        flags[0] = c + 1;
      }
    }
    ok = __syncthreads_and(ok);
  }
  const int last = nchunks - 1;
  if (ok) ok = __syncthreads_and(wait_bounded(bar_done + 8 * (last & 1), (last >> 1) & 1, a.err));

  if (ok) {
    tc_after();
    const int quad = warp & 3, colh = warp >> 2;
    const int i = i0 + 32 * quad + lane;
    for (int c0 = 64 * colh; c0 < min(nmma, 64 * colh + 64); c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + c0, v);
      if (i < a.dv) {
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const int t = c0 + cc;
          if (t < ntok)
            a.o[((size_t)(n0 + t) * a.H + h) * a.dv + i] = __float2bfloat16_rn(__uint_as_float(v[cc]));
        }
      }
    }
  }

  tc_before();
  __syncthreads();
  tc_after();
  if (!ok) {
    const int committed = flags[0], loaded = flags[1];
    // the copies of a chunk that never reached its MMAs, and the MMAs of the last commit
    if (threadIdx.x == 0 && loaded > committed) {
      const int c = loaded - 1;
      drain_bounded(bar_full + 8 * (c & 1), (c >> 1) & 1, a.err);
    }
    if (threadIdx.x == 32 && committed > 0) {
      const int c = committed - 1;
      drain_bounded(bar_done + 8 * (c & 1), (c >> 1) & 1, a.err);
    }
    __syncthreads();
  }
  if (warp == 1) tmem_free_cols(tmem);
}

// Tokens per CTA of the absorbed query: enough token tiles that the grid covers the 148 SMs
// about twice, each a multiple of 16 (the MMA's N step) and at most max_tile (the TMEM
// accumulator's 128 columns).
int token_tile(int n, int ctas_per_tile, int max_tile) {
  const int want = (2 * 148 + ctas_per_tile - 1) / ctas_per_tile;
  int tiles = (n + max_tile - 1) / max_tile;
  tiles = std::max(tiles, std::min(want, (n + 15) / 16));
  return std::min(max_tile, round_up((n + tiles - 1) / tiles, 16));
}

size_t absorb_smem(int dh, int dr, int tile) {
  const size_t need = 1024 + 2 * (size_t)dh * 128 +
                      (size_t)(dh / kSlab) * round_up(tile * 128, 1024) + 64 + 8 * (size_t)dr;
  // at least 51 KB: no more than four CTAs (4 x 128 TMEM columns) share an SM
  return std::max(need, (size_t)51 * 1024);
}

size_t output_smem(int tile) {
  const size_t stage = 2 * (size_t)kWRows * 128 + 4 * (size_t)round_up(tile * 128, 1024);
  return std::max((size_t)1024 + 2 * stage + 64, (size_t)80 * 1024);
}

}  // namespace

bool absorb_tc_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.head_dim % kSlab == 0 && c.head_dim <= 256 &&
         c.kv_rank % kSlab == 0 && c.rope_dim % 8 == 0;
}

bool output_tc_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.kv_rank % kSlab == 0;
}

cudaError_t launch_absorb_tc(const mla_config& c, const void* q_nope, const void* q_rope,
                             const int32_t* pos, const void* w_uk, void* q_out, int n,
                             uint32_t* err, cudaStream_t st) {
  const int H = c.num_heads, dh = c.head_dim, r = c.kv_rank;
  const int jts = (r + kWRows - 1) / kWRows;
  const int tile = token_tile(n, jts * H, kMaxTokTile);
  CUtensorMap tw, tq;
  if (!make_bf16_map(&tw, w_uk, (uint64_t)r, (uint64_t)H * dh, (uint64_t)r * 2, (uint32_t)dh) ||
      !make_bf16_map(&tq, q_nope, (uint64_t)H * dh, (uint64_t)n, (uint64_t)H * dh * 2,
                     (uint32_t)tile))
    return cudaErrorInvalidValue;
  const size_t smem = absorb_smem(dh, c.rope_dim, tile);
  cudaError_t e = cudaFuncSetAttribute(absorb_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  AbsorbArgs a{(const __nv_bfloat16*)q_rope, pos, (__nv_bfloat16*)q_out, err, n, H, dh, r,
               c.rope_dim, tile, c.rope_base};
  dim3 grid((n + tile - 1) / tile, jts, H);
  return launch_pdl(absorb_tc_kernel, grid, dim3(128), smem, st, tw, tq, a);
}

cudaError_t launch_output_tc(const mla_config& c, const float* lat, const void* w_uv, void* o,
                             int n, uint32_t* err, cudaStream_t st) {
  const int H = c.num_heads, dv = c.head_dim_v, r = c.kv_rank;
  const int mts = (dv + kWRows - 1) / kWRows;
  // every MMA instruction costs about the same whatever its N, and a CTA issues 2 r/16 of them
  // (hi and lo terms), so the tokens are split over CTAs only as far as needed to keep each
  // CTA's N at 128 or less
  // (up to 64 tokens, two CTAs per head fill the SMs better than one)
  const int tiles = n <= 64 ? (n + 31) / 32 : (n + kOutTokTile - 1) / kOutTokTile;
  const int tile = std::min(kOutTokTile, round_up((n + tiles - 1) / tiles, 16));
  if (((uintptr_t)lat & 15) != 0) return cudaErrorInvalidValue;
  CUtensorMap tw;
  if (!make_bf16_map(&tw, w_uv, (uint64_t)r, (uint64_t)H * dv, (uint64_t)r * 2, kWRows))
    return cudaErrorInvalidValue;
  const size_t smem = output_smem(tile);
  cudaError_t e = cudaFuncSetAttribute(output_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  OutputArgs a{lat, (__nv_bfloat16*)o, err, n, H, dv, r, tile};
  dim3 grid((n + tile - 1) / tile, mts, H);
  return launch_pdl(output_tc_kernel, grid, dim3(256), smem, st, tw, a);
}

cudaError_t launch_step_prep(const mla_config& c, const void* q_nope, const void* q_rope,
                             const int32_t* pos, const void* w_uk, void* q_out, int n,
                             const void* ckv, const void* kr, const float* gamma,
                             const int32_t* seq, const DecodeParams& p, void* pool,
                             cudaStream_t st) {
  const int H = c.num_heads, dh = c.head_dim, r = c.kv_rank;
  const int jts = (r + kWRows - 1) / kWRows;
  const int tile = token_tile(n, jts * H, kMaxTokTile);
  CUtensorMap tw, tq;
  if (!make_bf16_map(&tw, w_uk, (uint64_t)r, (uint64_t)H * dh, (uint64_t)r * 2, (uint32_t)dh) ||
      !make_bf16_map(&tq, q_nope, (uint64_t)H * dh, (uint64_t)n, (uint64_t)H * dh * 2,
                     (uint32_t)tile))
    return cudaErrorInvalidValue;
  const size_t smem = absorb_smem(dh, c.rope_dim, tile);
  cudaError_t e = cudaFuncSetAttribute(step_prep_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  PrepArgs a;
  a.ab = AbsorbArgs{(const __nv_bfloat16*)q_rope, pos, (__nv_bfloat16*)q_out, p.err, n, H, dh, r,
                    c.rope_dim, tile, c.rope_base};
  a.ax = (n + tile - 1) / tile;
  a.ay = jts;
  a.az = H;
  a.ckv = (const __nv_bfloat16*)ckv;
  a.kr = (const __nv_bfloat16*)kr;
  a.gamma = gamma;
  a.seq = seq;
  a.pool = (__nv_bfloat16*)pool;
  a.app_ctas = (n + kPrepThreads / 32 - 1) / (kPrepThreads / 32);
  a.eps = c.rms_eps;
  a.vec = c.kv_rank % 256 == 0 && c.kv_rank <= 1024 && ((uintptr_t)ckv & 15) == 0 &&
          ((uintptr_t)gamma & 15) == 0 && ((uintptr_t)pool & 15) == 0 &&
          ((c.kv_rank + c.rope_dim) * 2) % 16 == 0;
  a.p = p;
  const int grid = 1 + a.app_ctas + a.ax * a.ay * a.az;
  return launch_pdl(step_prep_kernel, dim3(grid), dim3(kPrepThreads), smem, st, tw, tq, a);
}

}  // namespace mla
