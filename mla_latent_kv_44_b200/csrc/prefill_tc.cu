// MLA prefill: causal attention of a prompt's tokens over themselves, in the expanded form,
// for sm_100a.
//   K_nope[j, h] = W_UK[h] c_kv[j],  V[j, h] = W_UV[h] c_kv[j]           ("MLA from scratch in
//   s = scale * ([q_nope ‖ RoPE(q_rope)] . [K_nope ‖ k_rope]),            PyTorch", The
//   query i attends keys 0 .. i of its sequence, o = softmax(s) V          MLAAttention module:
//                                                                         K and V rebuilt from
// the latent, the causal mask over the S > 1 new tokens). With many queries per key the
// expanded form costs fewer FLOPs than the absorbed one (d_h + d_r = 192 per score against
// r + d_r = 576), so K and V are expanded once per key, by a persistent tensor-core GEMM that
// keeps a 128-row weight tile in shared memory and streams the tokens' c_kv (read in place
// from the cache rows); other shapes use the front end's split-K weight stream. A pack kernel
// rotates the query's RoPE part (angles in double); the attention reads q_nope where the
// caller keeps it.
// The attention kernel takes one CTA per (two adjacent 128-query tiles A and B, head) of a
// sequence (DeepSeek-V2's head shape: d_h = 128, d_r = 64, d_v = 128, bf16), longest pairs
// first. Both query tiles stay in shared memory and share every key and value tile TMA brings
// (K_nope of the head and the shared k_rope: three 64-wide slabs through a ring of four; V: two
// slabs, double-buffered). One MMA warp issues, per key tile j, O_A += P_A V_j,
// S_A = Q_A K_{j+1}^T, O_B += P_B V_j, S_B = Q_B K_{j+1}^T (M = 128 queries, N = 128 keys or
// values; S from shared memory, P read from TMEM: the TS form), the whole warp waiting and one
// elected lane issuing. Two groups of four warps take a tile each (a thread per query row):
// row maximum, rescale of O in TMEM when the maximum grows by more than 2^8, exp2 (one pair in
// eight on the FMA pipe), P in bf16 written back over the tile's S columns. While one group's
// softmax runs the tensor core works on the other tile's products. Key tiles above a query
// tile's diagonal are skipped; the diagonal tile is masked. Other shapes and fp32 take a
// CUDA-core kernel (a warp per (query, head), online softmax over the keys).
// Every mbarrier wait gives up after 1 s: the kernel then sets MLA_DEV_WAIT_TIMEOUT, waits
// (bounded) for what it issued, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_map.h"

namespace mla {

size_t front_part_bytes(const mla_config& c, int K, int n, const int* rows, int nseg,
                        bool norm);
cudaError_t launch_front_linear(const mla_config& c, const void* x, int n, int K, int ldx,
                                const void* const* w, const int* rows, void* const* out, int nseg,
                                int norm_seg, const float* gamma, float eps, void* part,
                                uint32_t* err, cudaStream_t st);

namespace {

constexpr unsigned long long kPfTimeoutNs = 1000000000ull;
constexpr int kPfTile = 128;                   // queries per tile = keys per tile
constexpr int kPfSlabBytes = kPfTile * 128;    // 128 rows x 64 bf16: 16 KB
constexpr int kPfQ = 0;                        // two query tiles: 3 slabs each (q_nope 0-63,
                                               // 64-127, q_rope)
constexpr int kPfK = kPfQ + 6 * kPfSlabBytes;  // keys: a ring of 4 slabs; key tile j's slab s
                                               // (K_nope 0-63, 64-127, k_rope) in slot
                                               // (3j + s) % 4
constexpr int kPfKSlots = 4;
constexpr int kPfV = kPfK + kPfKSlots * kPfSlabBytes;  // values: 2 stages of 2 slabs (d_v 0-63,
                                                       // 64-127), MN-major
constexpr int kPfBar = kPfV + 4 * kPfSlabBytes;
constexpr int kPfSmem = kPfBar + 256 + 1024;
constexpr int kPfThreads = 320;                // warps 0-3, 4-7: softmax of tiles A, B;
                                               // 8: TMA; 9: MMA issue
constexpr uint32_t kPfTmemCols = 512;          // S_A, S_B, O_A, O_B: 128 columns each

__device__ __forceinline__ bool pf_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > kPfTimeoutNs) {
      set_error(err, MLA_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 2^x for a pair on the FMA pipe, so that the exp2 unit and the FMA pipe share a tile's
// exponentials: Cody and Waite's reduction x = k + f with k = round(x) and f in [-1/2, 1/2]
// (k from adding 1.5 * 2^23, which leaves it in the low mantissa bits), 2^f by a cubic fitted
// to the relative error on [-1/2, 1/2] (at most 7.5e-5, against 2^-9 for the bf16 rounding of
// P that follows), and k added to the exponent field as an integer. Arguments below -126
// (masked keys' -inf included) are clamped there; their 2^x is below 2^-125 instead of 0.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 k = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(k, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(f, make_float2(0.05517132f, 0.05517132f),
                        make_float2(0.24261054f, 0.24261054f));
  p = __ffma2_rn(p, f, make_float2(0.69326097f, 0.69326097f));
  p = __ffma2_rn(p, f, make_float2(0.99992812f, 0.99992812f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// tcgen05 issue from a converged warp: every lane runs the issue loop, so the descriptors stay
// warp-uniform, and elect.sync picks the one lane that issues.
__device__ __forceinline__ void mma_ss_warp(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t id,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d), "l"(adesc),
      "l"(bdesc), "r"(id), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts_warp(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t id,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d), "r"(a),
      "l"(bdesc), "r"(id), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit_warp(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}

// Pairs of a row's 64 whose exponentials go to the FMA pipe: (pair % 8) < kPfFmaEighths.
constexpr int kPfFmaEighths = 1;

// Warp-wide bounded wait: the same result in every lane.
__device__ __forceinline__ bool warp_all_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
  bool done = false, ok = true;
  const uint64_t t0 = globaltimer();
  while (true) {
    done = __all_sync(0xffffffffu, mbar_try(bar, parity));
    if (done) break;
    if (__any_sync(0xffffffffu, globaltimer() - t0 > kPfTimeoutNs)) {
      if ((threadIdx.x & 31) == 0) set_error(err, MLA_DEV_WAIT_TIMEOUT);
      ok = false;
      break;
    }
  }
  return ok;
}

// The sequence of token index i: cu_seqlens[b] <= i < cu_seqlens[b + 1] (binary search).
__device__ __forceinline__ int seq_of(const int32_t* cu, int batch, int i) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= i) lo = mid; else hi = mid;
  }
  return lo;
}

// Q = [q_nope ‖ RoPE(q_rope, pos)] per (token, head): grid (tokens), 16-byte pieces (VEC
// values) per thread: q_nope pieces copied, q_rope pieces rotated pair by pair (angle and
// rotation in double, rounded once). With rope_only, q holds just the rotated RoPE part
// (n, H, d_r): the tensor-core attention reads q_nope where the caller keeps it.
template <typename T>
__global__ void __launch_bounds__(256)
prefill_pack_kernel(const T* q_nope, const T* q_rope, const int32_t* pos, T* q, int H, int dh,
                    int dr, float base, bool rope_only) {
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ double cs[];  // [2][dr / 2]: cos, sin of the token's angles
  const int n = blockIdx.x, half = dr / 2;
  const int pn = dh / VEC, pr = dr / VEC;  // pieces per head
  const int skip = rope_only ? pn : 0, pd = pn + pr - skip, D = rope_only ? dr : dh + dr;
  wait_prior_grid();
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    rope_cos_sin(pos[n], i, dr, base, &cs[i], &cs[half + i]);
  __syncthreads();
  for (int e = threadIdx.x; e < H * pd; e += blockDim.x) {
    const int h = e / pd, c = e - h * pd + skip;
    uint4 out;
    if (c < pn) {
      out = *(const uint4*)(q_nope + ((size_t)n * H + h) * dh + c * VEC);
    } else {
      const int k0 = (c - pn) * VEC;  // first rope value of the piece (even)
      const uint4 in = *(const uint4*)(q_rope + ((size_t)n * H + h) * dr + k0);
      const T* x = (const T*)&in;
      T* y = (T*)&out;
#pragma unroll
      for (int u = 0; u < VEC; u += 2) {
        const int i = (k0 + u) >> 1;
        const double x0 = to_f32(x[u]), x1 = to_f32(x[u + 1]);
        y[u] = from_f32<T>((float)(x0 * cs[i] - x1 * cs[half + i]));
        y[u + 1] = from_f32<T>((float)(x0 * cs[half + i] + x1 * cs[i]));
      }
    }
    *(uint4*)(q + ((size_t)n * H + h) * D + (c - skip) * VEC) = out;
  }
}

struct PrefillArgs {
  const int32_t* cu;
  __nv_bfloat16* o;
  uint32_t* err;
  int batch, H, pairs;  // pairs: query-tile pairs per sequence in the grid (max_seqlen / 256)
  float c2;             // softmax scale * log2(e)
};

// Grid (batch * pairs, H); 320 threads. TMA maps: qn (n, H * 128) the caller's q_nope, qr
// (n, H * 64) the rotated RoPE query, kn (n, H * 128), rows (n, r + 64): k_rope at column r,
// v (n, H * 128); all with 128-row boxes of 64 columns.
__global__ void __launch_bounds__(kPfThreads)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qr,
                  const __grid_constant__ CUtensorMap tm_kn,
                  const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_v,
                  const PrefillArgs a, int r) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = saddr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a sequence's pairs of query tiles, longest first, so that the grid's last CTAs are short
  const int b = blockIdx.x / a.pairs, pr = a.pairs - 1 - (blockIdx.x - b * a.pairs);
  const int h = blockIdx.y;
  // barriers: q, kfull[4], kfree[4], vfull[2], vfree[2], s[2], p[2], o[2], final
  const uint32_t bar_q = sb + kPfBar, bar_kfull = bar_q + 8, bar_kfree = bar_q + 40;
  const uint32_t bar_vfull = bar_q + 72, bar_vfree = bar_q + 88;
  const uint32_t bar_s = bar_q + 104, bar_p = bar_q + 120, bar_o = bar_q + 136;
  const uint32_t bar_fin = bar_q + 152;
  uint32_t* tmem_slot = (uint32_t*)(smem + kPfBar + 160);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 20; ++i) mbar_init(bar_q + 8 * i, (i == 15 || i == 16) ? 4 : 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(kPfTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  wait_prior_grid();
  const int start = a.cu[b], len = a.cu[b + 1] - start;
  const int q0 = pr * 2 * kPfTile;
  // key tiles of each query tile: 0 .. its diagonal (none when the tile starts past the end)
  int nkt[2];
  for (int g = 0; g < 2; ++g) {
    const int qg = q0 + g * kPfTile;
    nkt[g] = qg < len ? (min(len, qg + kPfTile) - 1) / kPfTile + 1 : 0;
  }
  const int nk = max(nkt[0], nkt[1]);  // tile B's count when it has rows
  bool ok = true;
  if (nkt[0] > 0) {
    if (warp == 8) {
      // ---------------------------------------------------------------- TMA
      // in the order the MMA warp consumes them: key tile j's first slab, its values, then its
      // other two slabs (their slots are freed by the second score product of tile j - 1)
      if (lane == 0) {
        const int ntile = nkt[1] > 0 ? 2 : 1;
        mbar_expect_tx(bar_q, 3 * kPfSlabBytes * ntile);
        for (int g = 0; g < ntile; ++g)
          for (int s = 0; s < 3; ++s)
            tma_load(sb + kPfQ + (3 * g + s) * kPfSlabBytes, s < 2 ? &tm_qn : &tm_qr, bar_q,
                     s < 2 ? h * 128 + 64 * s : h * 64, start + q0 + g * kPfTile);
        int k_issued = 0, v_issued = 0;  // slabs and value tiles issued
        auto load_k = [&](int j, int sl) {
          const int u = 3 * j + sl, slot = u & (kPfKSlots - 1);
          if (u >= kPfKSlots && !pf_wait(bar_kfree + 8 * slot, ((u >> 2) - 1) & 1, a.err))
            return false;
          mbar_expect_tx(bar_kfull + 8 * slot, kPfSlabBytes);
          if (sl < 2)
            tma_load(sb + kPfK + slot * kPfSlabBytes, &tm_kn, bar_kfull + 8 * slot,
                     h * 128 + 64 * sl, start + j * kPfTile);
          else
            tma_load(sb + kPfK + slot * kPfSlabBytes, &tm_kr, bar_kfull + 8 * slot, r,
                     start + j * kPfTile);
          k_issued = u + 1;
          return true;
        };
        for (int j = 0; j < nk && ok; ++j) {
          ok = load_k(j, 0);
          if (!ok) break;
          const int vs = j & 1;
          if (j >= 2) ok = pf_wait(bar_vfree + 8 * vs, ((j >> 1) - 1) & 1, a.err);
          if (!ok) break;
          mbar_expect_tx(bar_vfull + 8 * vs, 2 * kPfSlabBytes);
          for (int s = 0; s < 2; ++s)
            tma_load(sb + kPfV + (2 * vs + s) * kPfSlabBytes, &tm_v, bar_vfull + 8 * vs,
                     h * 128 + 64 * s, start + j * kPfTile);
          v_issued = j + 1;
          ok = load_k(j, 1) && load_k(j, 2);
        }
        // the last copies have landed before the CTA may exit (each barrier's last armed phase
        // is its last, so the wait holds whether or not a consumer saw it)
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar_q, 0) && globaltimer() - t0 < kPfTimeoutNs) {
        }
        for (int u = max(0, k_issued - kPfKSlots); u < k_issued; ++u)
          while (!mbar_try(bar_kfull + 8 * (u & (kPfKSlots - 1)), (u >> 2) & 1) &&
                 globaltimer() - t0 < 2 * kPfTimeoutNs) {
          }
        for (int j = max(0, v_issued - 2); j < v_issued; ++j)
          while (!mbar_try(bar_vfull + 8 * (j & 1), (j >> 1) & 1) &&
                 globaltimer() - t0 < 3 * kPfTimeoutNs) {
          }
      }
    } else if (warp == 9) {
      // ---------------------------------------------------------------- MMA issue
      // Per key tile j: O_A += P_A V_j, S_A = Q_A K_{j+1}^T, O_B += P_B V_j, S_B = Q_B K_{j+1}^T,
      // so that each tile's next scores are computed while the other tile's softmax runs. The
      // whole warp runs the loop and waits warp-wide; one elected lane issues.
      {
        const uint32_t id_s = idesc(128, 128, 0, 0), id_o = idesc(128, 128, 1);
        // S_g = Q_g K_j^T; the last product to read key tile j frees its slabs one by one
        auto scores = [&](int g, int j) {
          const bool last = g == 1 || nkt[1] <= j;
          for (int sl = 0; sl < 3; ++sl) {
            const int u = 3 * j + sl, slot = u & (kPfKSlots - 1);
            if (!warp_all_wait(bar_kfull + 8 * slot, (u >> 2) & 1, a.err)) return false;
            tc_after();
            for (int kk = 0; kk < 4; ++kk)
              mma_ss_warp(tmem + 128 * g,
                          sdesc(sb + kPfQ + (3 * g + sl) * kPfSlabBytes + 32u * kk, 16, 1024, 2),
                          sdesc(sb + kPfK + slot * kPfSlabBytes + 32u * kk, 16, 1024, 2), id_s,
                          (sl | kk) ? 1u : 0u);
            if (last) commit_warp(bar_kfree + 8 * slot);
          }
          commit_warp(bar_s + 8 * g);
          return true;
        };
        ok = warp_all_wait(bar_q, 0, a.err) && scores(0, 0) && (nkt[1] == 0 || scores(1, 0));
        for (int j = 0; j < nk && ok; ++j) {
          const int vs = j & 1;
          ok = warp_all_wait(bar_vfull + 8 * vs, (j >> 1) & 1, a.err);
          for (int g = 0; g < 2 && ok; ++g) {
            if (j >= nkt[g]) continue;
            ok = warp_all_wait(bar_p + 8 * g, j & 1, a.err);
            if (!ok) break;
            tc_after();
            for (int ks = 0; ks < 8; ++ks)  // 16 keys per step: 8 TMEM columns of P
              mma_ts_warp(tmem + 256 + 128 * g, tmem + 128 * g + 8 * ks,
                          sdesc(sb + kPfV + 2 * vs * kPfSlabBytes + 2048u * (uint32_t)ks,
                                kPfSlabBytes, 1024, 2),
                          id_o, (j > 0 || ks > 0) ? 1u : 0u);
            commit_warp(bar_o + 8 * g);
            if (g == 1 || nkt[1] <= j) commit_warp(bar_vfree + 8 * vs);  // V_j's last reader
            // S_g's columns hold P_g until its P . V is done
            if (j + 1 < nkt[g])
              ok = warp_all_wait(bar_o + 8 * g, j & 1, a.err) && scores(g, j + 1);
          }
        }
      }
    } else if (nkt[warp >> 2] > 0) {
      // ---------------------------------------------------------------- softmax of tile g
      const int g = warp >> 2, quad = warp & 3;
      const int row = quad * 32 + lane;          // TMEM lane = query row within the tile
      const int qi = q0 + g * kPfTile + row;     // query index within the sequence
      const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
      const uint32_t t_s = tmem + lane_base + 128 * g, t_o = tmem + lane_base + 256 + 128 * g;
      float m_ref = 0.f, l = 0.f;
      for (int j = 0; j < nkt[g] && ok; ++j) {
        ok = warp_all_wait(bar_s + 8 * g, j & 1, a.err);
        if (!ok) break;
        tc_after();
        uint32_t v[128];
        tmem_ld128(t_s, v);
        // the last key tile is the diagonal one (it starts at the query tile's first row):
        // keys past the row's query are masked there; earlier tiles are visible whole
        if (j == nkt[g] - 1) {
          const int lim = row;  // keys 0 .. row of the tile are visible
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) v[c] = 0xff800000u;  // -inf
        }
        // the row maximum of the raw scores (the scale is positive), four three-input chains
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int k = 0; k < 128; k += 8)
#pragma unroll
          for (int c = 0; c < 4; ++c)
            mx4[c] = fmax3(mx4[c], __uint_as_float(v[k + 2 * c]), __uint_as_float(v[k + 2 * c + 1]));
        const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * a.c2;
        float alpha = 1.f;
        if (j == 0) {
          m_ref = qi < len ? mx : 0.f;  // key 0 is visible to every query of the sequence
        } else if (mx > m_ref + 8.f) {
          alpha = ex2(m_ref - mx);
          m_ref = mx;
        }
        // P = exp2(s * c2 - m_ref) in bf16 over the tile's S columns (keys 2c, 2c + 1 in
        // column c), the argument two at a time in one packed fma, one pair in eight on the
        // FMA pipe; l sums the bf16 values the MMA consumes, two at a time in packed adds
        const float2 c2x2 = make_float2(a.c2, a.c2), nm = make_float2(-m_ref, -m_ref);
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float2 x = __ffma2_rn(
              make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), c2x2, nm);
          const float2 e = (c & 7) < kPfFmaEighths ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
          v[c] = pack_bf16(e.x, e.y);
          rs2[c & 1] = __fadd2_rn(
              rs2[c & 1], make_float2(__uint_as_float(v[c] << 16), __uint_as_float(v[c] & 0xffff0000u)));
        }
        const float rs = (rs2[0].x + rs2[1].x) + (rs2[0].y + rs2[1].y);
        l = l * alpha + rs;
        // the previous P . V is complete (S_g of this tile was issued after it): rescale O
        // (TMEM accesses are warp-wide: a warp rescales when any of its rows must)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(t_o + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + c0, o);
          }
        }
        uint32_t w0[32], w1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          w0[i] = v[i];
          w1[i] = v[32 + i];
        }
        tmem_st32(t_s, w0);
        tmem_st32(t_s + 32, w1);
        tmem_wait_st();
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p + 8 * g);
      }
      if (ok) ok = warp_all_wait(bar_o + 8 * g, (nkt[g] - 1) & 1, a.err);
      if (ok) {
        tc_after();
        // o = O / l for this thread's query row, bf16 (every lane takes part in the warp-wide
        // TMEM loads; rows past the sequence end store nothing)
        const float inv = qi < len ? 1.f / l : 0.f;
        __nv_bfloat16* dst = a.o + ((size_t)(start + min(qi, len - 1)) * a.H + h) * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(t_o + c0, o);
          if (qi < len) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
              *(uint4*)(dst + c0 + i) = w;
            }
          }
        }
      }
    }
  }
  __syncwarp();
  tc_before();
  __syncthreads();
  tc_after();
  if (threadIdx.x == 9 * 32) {
    // every MMA issued here (none when the work was empty) is done before TMEM is freed; the
    // copies issued were all waited for by the MMA thread unless a wait gave up, in which case
    // the last ones get a bounded wait too
    tc_commit(bar_fin);
    const uint64_t t0 = globaltimer();
    while (!mbar_try(bar_fin, 0) && globaltimer() - t0 < kPfTimeoutNs) {
    }
  }
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kPfTmemCols)
                 : "memory");
}

// K_nope = c_kv W_UK^T and V = c_kv W_UV^T for every prompt token on the tensor cores, one
// GEMM with M = 128 tokens, N = 128 weight rows, K = r per tile. A persistent CTA per SM walks
// work items (a 128-row weight tile, a chunk of token tiles): the weight tile stays in shared
// memory (r / 64 slabs of 16 KB, each replaced for the next item as soon as the item's last
// products are done with it) while the tokens' c_kv slabs stream through a ring; two TMEM
// accumulators let the epilogue of one token tile (bf16, a thread per token writing the tile's
// 128 contiguous outputs) overlap the products of the next. Warps: 0 TMA, 1 MMA issue (whole
// warp, one elected lane), 2-5 epilogue.
constexpr int kExSlab = 128 * 128;             // 128 rows x 64 bf16: 16 KB
constexpr int kExMaxSlabs = 8;                 // resident weight tile: r <= 512
constexpr int kExStages = 6;                   // token slabs in flight
constexpr int kExW = 0;
constexpr int kExX = kExW + kExMaxSlabs * kExSlab;
constexpr int kExBar = kExX + kExStages * kExSlab;
constexpr int kExSmem = kExBar + 512 + 1024;
constexpr int kExThreads = 192;
constexpr int kExChunk = 16;                   // token tiles per work item

struct ExpandArgs {
  __nv_bfloat16* kn;
  __nv_bfloat16* v;
  uint32_t* err;
  int n;              // tokens
  int ksl;            // 64-wide slabs of r
  int mt_k, mtiles;   // 128-row weight tiles of W_UK; of W_UK and W_UV together
  int chunks, items;  // token chunks per weight tile; work items
  int ldk, ldv;       // output row pitches (elements)
};

__global__ void __launch_bounds__(kExThreads)
expand_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wk,
                 const __grid_constant__ CUtensorMap tm_wv, const ExpandArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = saddr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers: wfull[8], wfree[8], xfull[6], xfree[6], afull[2], afree[2], final
  const uint32_t bar_wfull = sb + kExBar, bar_wfree = bar_wfull + 8 * kExMaxSlabs;
  const uint32_t bar_xfull = bar_wfree + 8 * kExMaxSlabs, bar_xfree = bar_xfull + 8 * kExStages;
  const uint32_t bar_afull = bar_xfree + 8 * kExStages, bar_afree = bar_afull + 16;
  const uint32_t bar_fin = bar_afree + 16;
  uint32_t* tmem_slot = (uint32_t*)(smem + kExBar + 320);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * kExMaxSlabs + 2 * kExStages + 4 + 1; ++i) {
      const uint32_t b = bar_wfull + 8 * i;
      mbar_init(b, (b == bar_afree || b == bar_afree + 8) ? 4 : 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(256)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  wait_prior_grid();
  const int ttiles = (a.n + 127) / 128;
  bool ok = true;
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      int kx = 0, li = 0;
      for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x, ++li) {
        const int mt = it / a.chunks, tt0 = (it - mt * a.chunks) * kExChunk;
        const int tt1 = min(ttiles, tt0 + kExChunk);
        const bool uk = mt < a.mt_k;
        for (int tt = tt0; tt < tt1 && ok; ++tt)
          for (int s = 0; s < a.ksl; ++s, ++kx) {
            if (tt == tt0) {
              // weight slab s, once the previous item's last products are done with it
              if (li > 0 && !pf_wait(bar_wfree + 8 * s, (li - 1) & 1, a.err)) {
                ok = false;
                break;
              }
              mbar_expect_tx(bar_wfull + 8 * s, kExSlab);
              tma_load(sb + kExW + s * kExSlab, uk ? &tm_wk : &tm_wv, bar_wfull + 8 * s, 64 * s,
                       (uk ? mt : mt - a.mt_k) * 128);
            }
            const int st = kx % kExStages, use = kx / kExStages;
            if (use > 0 && !pf_wait(bar_xfree + 8 * st, (use - 1) & 1, a.err)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar_xfull + 8 * st, kExSlab);
            tma_load(sb + kExX + st * kExSlab, &tm_x, bar_xfull + 8 * st, 64 * s, tt * 128);
          }
      }
      // the last copies have landed before the CTA may exit
      const uint64_t t0 = globaltimer();
      for (int s = 0; s < a.ksl && li > 0; ++s)
        while (!mbar_try(bar_wfull + 8 * s, (li - 1) & 1) && globaltimer() - t0 < kPfTimeoutNs) {
        }
      for (int u = max(0, kx - kExStages); u < kx; ++u)
        while (!mbar_try(bar_xfull + 8 * (u % kExStages), (u / kExStages) & 1) &&
               globaltimer() - t0 < 2 * kPfTimeoutNs) {
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t id = idesc(128, 128, 0, 0);
    int kx = 0, tcount = 0, li = 0;
    for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x, ++li) {
      const int mt = it / a.chunks, tt0 = (it - mt * a.chunks) * kExChunk;
      const int tt1 = min(ttiles, tt0 + kExChunk);
      for (int tt = tt0; tt < tt1 && ok; ++tt, ++tcount) {
        const int acc = tcount & 1;
        // the accumulator's previous tile has been read out by the epilogue
        if (tcount >= 2) ok = warp_all_wait(bar_afree + 8 * acc, ((tcount >> 1) - 1) & 1, a.err);
        for (int s = 0; s < a.ksl && ok; ++s, ++kx) {
          const int st = kx % kExStages;
          if (tt == tt0) ok = warp_all_wait(bar_wfull + 8 * s, li & 1, a.err);
          ok = ok && warp_all_wait(bar_xfull + 8 * st, (kx / kExStages) & 1, a.err);
          if (!ok) break;
          tc_after();
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_warp(tmem + 128 * acc, sdesc(sb + kExX + st * kExSlab + 32u * kk, 16, 1024, 2),
                        sdesc(sb + kExW + s * kExSlab + 32u * kk, 16, 1024, 2), id,
                        (s | kk) ? 1u : 0u);
          commit_warp(bar_xfree + 8 * st);
          if (tt == tt1 - 1) commit_warp(bar_wfree + 8 * s);  // the item's last read of slab s
        }
        if (ok) commit_warp(bar_afull + 8 * acc);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    int tcount = 0;
    for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
      const int mt = it / a.chunks, tt0 = (it - mt * a.chunks) * kExChunk;
      const int tt1 = min(ttiles, tt0 + kExChunk);
      const bool uk = mt < a.mt_k;
      __nv_bfloat16* out = uk ? a.kn : a.v;
      const int ld = uk ? a.ldk : a.ldv, col0 = (uk ? mt : mt - a.mt_k) * 128;
      for (int tt = tt0; tt < tt1 && ok; ++tt, ++tcount) {
        const int acc = tcount & 1;
        ok = warp_all_wait(bar_afull + 8 * acc, (tcount >> 1) & 1, a.err);
        if (!ok) break;
        tc_after();
        const int token = tt * 128 + quad * 32 + lane;
        __nv_bfloat16* dst = out + (size_t)min(token, a.n - 1) * ld + col0;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t x[32];
          tmem_ld32(tmem + lane_base + 128 * acc + c0, x);
          if (token < a.n) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(x[i]), __uint_as_float(x[i + 1]));
              w.y = pack_bf16(__uint_as_float(x[i + 2]), __uint_as_float(x[i + 3]));
              w.z = pack_bf16(__uint_as_float(x[i + 4]), __uint_as_float(x[i + 5]));
              w.w = pack_bf16(__uint_as_float(x[i + 6]), __uint_as_float(x[i + 7]));
              *(uint4*)(dst + c0 + i) = w;
            }
          }
        }
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afree + 8 * acc);
      }
    }
  }
  __syncwarp();
  tc_before();
  __syncthreads();
  tc_after();
  if (threadIdx.x == 32) {
    // every MMA issued here is done before TMEM is freed
    tc_commit(bar_fin);
    const uint64_t t0 = globaltimer();
    while (!mbar_try(bar_fin, 0) && globaltimer() - t0 < kPfTimeoutNs) {
    }
  }
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256)
                 : "memory");
}

// CUDA-core prefill: a warp per (query, head); lanes split the score's dims and the value's.
template <typename T>
__global__ void __launch_bounds__(128)
prefill_simt_kernel(const T* q, const T* kn, const T* rows, const T* v, const int32_t* cu,
                    int batch, int H, int dh, int dr, int dv, int ldr, int r, float c2, T* o) {
  const int i = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 4 + warp;
  wait_prior_grid();
  if (h >= H) return;
  const int b = seq_of(cu, batch, i), start = cu[b];
  const int D = dh + dr;
  const T* qr = q + ((size_t)i * H + h) * D;
  float m = -INFINITY, l = 0.f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // d_v <= 256: lane's dims lane + 32u
  for (int j = start; j <= i; ++j) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float kd = d < dh ? to_f32(kn[((size_t)j * H + h) * dh + d])
                              : to_f32(rows[(size_t)j * ldr + r + (d - dh)]);
      s = fmaf(to_f32(qr[d]), kd, s);
    }
    s = warp_sum(s) * c2;
    const float mn = fmaxf(m, s);
    const float alpha = ex2(m - mn), p = ex2(s - mn);
    l = l * alpha + p;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int d = lane + 32 * u;
      const float vd = d < dv ? to_f32(v[((size_t)j * H + h) * dv + d]) : 0.f;
      acc[u] = fmaf(p, vd, acc[u] * alpha);
    }
    m = mn;
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int d = lane + 32 * u;
    if (d < dv) o[((size_t)i * H + h) * dv + d] = from_f32<T>(acc[u] / l);
  }
}

}  // namespace

bool prefill_tc_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.head_dim == 128 && c.rope_dim == 64 && c.head_dim_v == 128 &&
         c.kv_rank % 8 == 0;
}

// The expansion's tensor-core GEMM: bf16, the weight tile resident (r <= 512), whole 128-row
// weight tiles.
bool expand_tc_supported(const mla_config& c) {
  return prefill_tc_supported(c) && c.kv_rank <= 64 * kExMaxSlabs &&
         (c.num_heads * c.head_dim) % 128 == 0 && (c.num_heads * c.head_dim_v) % 128 == 0;
}

// Workspace: the query (n, H, d_r) rotated for the tensor cores, else (n, H, d_h + d_r)
// packed; K_nope (n, H * d_h), V (n, H * d_v) in dtype; then the front end's partial sums
// where its weight stream does the expansion.
struct PrefillLayout {
  size_t q, kn, v, part, total;
};

PrefillLayout prefill_layout(const mla_config& c, int n) {
  const size_t e = c.dtype == MLA_BF16 ? 2 : 4;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  PrefillLayout L;
  L.q = 0;
  // the tensor-core attention takes only the rotated RoPE part of the query from here
  const int qd = prefill_tc_supported(c) ? c.rope_dim : c.head_dim + c.rope_dim;
  L.kn = up((size_t)n * c.num_heads * qd * e);
  L.v = L.kn + up((size_t)n * c.num_heads * c.head_dim * e);
  L.part = L.v + up((size_t)n * c.num_heads * c.head_dim_v * e);
  // partial sums only for the front end's weight stream (the expansion GEMM writes K and V)
  const int rows[2] = {c.num_heads * c.head_dim, c.num_heads * c.head_dim_v};
  L.total = L.part + (expand_tc_supported(c)
                          ? 0
                          : up(front_part_bytes(c, c.kv_rank, n, rows, 2, false)));
  return L;
}

cudaError_t launch_prefill(const mla_config& c, const void* q_nope, const void* q_rope,
                           const int32_t* pos, const void* rows, const void* w_uk,
                           const void* w_uv, const int32_t* cu, int batch, int max_seqlen, int n,
                           void* o, void* ws, uint32_t* err, cudaStream_t st) {
  const int H = c.num_heads, dh = c.head_dim, dr = c.rope_dim, dv = c.head_dim_v,
            r = c.kv_rank;
  const PrefillLayout L = prefill_layout(c, n);
  uint8_t* w8 = (uint8_t*)ws;
  void* q = w8 + L.q;
  void* kn = w8 + L.kn;
  void* v = w8 + L.v;
  const bool bf = c.dtype == MLA_BF16, tc = prefill_tc_supported(c);
  // the rotated query: its RoPE part alone for the tensor cores, else packed with q_nope
  const size_t csm = (size_t)std::max(1, dr / 2) * 2 * sizeof(double);
  cudaError_t e = bf ? launch_pdl(prefill_pack_kernel<__nv_bfloat16>, dim3(n), dim3(256), csm, st,
                                  (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)q_rope, pos,
                                  (__nv_bfloat16*)q, H, dh, dr, c.rope_base, tc)
                     : launch_pdl(prefill_pack_kernel<float>, dim3(n), dim3(256), csm, st,
                                  (const float*)q_nope, (const float*)q_rope, pos, (float*)q, H,
                                  dh, dr, c.rope_base, false);
  if (e != cudaSuccess) return e;
  // K_nope and V from c_kv (the first r values of each cache row)
  if (expand_tc_supported(c)) {
    CUtensorMap tx, twk, twv;
    if (!make_bf16_map(&tx, rows, (uint64_t)r, (uint64_t)n, (uint64_t)(r + dr) * 2, 128) ||
        !make_bf16_map(&twk, w_uk, (uint64_t)r, (uint64_t)H * dh, (uint64_t)r * 2, 128) ||
        !make_bf16_map(&twv, w_uv, (uint64_t)r, (uint64_t)H * dv, (uint64_t)r * 2, 128))
      return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    e = cudaFuncSetAttribute(expand_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kExSmem);
    if (e != cudaSuccess) return e;
    const int ttiles = (n + 127) / 128, chunks = (ttiles + kExChunk - 1) / kExChunk;
    const int mt_k = H * dh / 128, mtiles = mt_k + H * dv / 128;
    ExpandArgs ea{(__nv_bfloat16*)kn, (__nv_bfloat16*)v, err, n, (r + 63) / 64, mt_k, mtiles,
                  chunks, mtiles * chunks, H * dh, H * dv};
    e = launch_pdl(expand_tc_kernel, dim3(std::min(sms, ea.items)), dim3(kExThreads),
                   (size_t)kExSmem, st, tx, twk, twv, ea);
  } else {
    const void* wts[2] = {w_uk, w_uv};
    const int wrows[2] = {H * dh, H * dv};
    void* outs[2] = {kn, v};
    e = launch_front_linear(c, rows, n, r, r + dr, wts, wrows, outs, 2, -1, nullptr, 0.f,
                            w8 + L.part, err, st);
  }
  if (e != cudaSuccess) return e;
  const float c2 = c.softmax_scale * 1.4426950408889634f;
  if (tc) {
    CUtensorMap tqn, tqr, tkn, tkr, tv;
    if (!make_bf16_map(&tqn, q_nope, (uint64_t)H * dh, (uint64_t)n, (uint64_t)H * dh * 2,
                       kPfTile) ||
        !make_bf16_map(&tqr, q, (uint64_t)H * dr, (uint64_t)n, (uint64_t)H * dr * 2, kPfTile) ||
        !make_bf16_map(&tkn, kn, (uint64_t)H * dh, (uint64_t)n, (uint64_t)H * dh * 2, kPfTile) ||
        !make_bf16_map(&tkr, rows, (uint64_t)(r + dr), (uint64_t)n, (uint64_t)(r + dr) * 2,
                       kPfTile) ||
        !make_bf16_map(&tv, v, (uint64_t)H * dv, (uint64_t)n, (uint64_t)H * dv * 2, kPfTile))
      return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPfSmem);
    if (e != cudaSuccess) return e;
    const int pairs = (max_seqlen + 2 * kPfTile - 1) / (2 * kPfTile);
    PrefillArgs a{cu, (__nv_bfloat16*)o, err, batch, H, pairs, c2};
    return launch_pdl(prefill_tc_kernel, dim3(batch * pairs, H), dim3(kPfThreads),
                      (size_t)kPfSmem, st, tqn, tqr, tkn, tkr, tv, a, r);
  }
  dim3 grid(n, (H + 3) / 4);
  return bf ? launch_pdl(prefill_simt_kernel<__nv_bfloat16>, grid, dim3(128), 0, st,
                         (const __nv_bfloat16*)q, (const __nv_bfloat16*)kn,
                         (const __nv_bfloat16*)rows, (const __nv_bfloat16*)v, cu, batch, H, dh,
                         dr, dv, r + dr, r, c2, (__nv_bfloat16*)o)
            : launch_pdl(prefill_simt_kernel<float>, grid, dim3(128), 0, st, (const float*)q,
                         (const float*)kn, (const float*)rows, (const float*)v, cu, batch, H, dh,
                         dr, dv, r + dr, r, c2, (float*)o);
}

size_t prefill_workspace_bytes(const mla_config& c, int n) { return prefill_layout(c, n).total; }

}  // namespace mla
