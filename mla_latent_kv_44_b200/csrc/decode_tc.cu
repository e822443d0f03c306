// tcgen05 tensor-core attention stage of mla_decode (bf16 cache, H = 128, r = 512, d_r = 64,
// 64-row cache blocks), for sm_100a.
//
// Absorbed decode ("DeepSeek MLA, Built From the Paper", 3 Matrix absorption; "Build a DeepSeek
// Model from Scratch" ch. 3, score = content score + position score; "MLA from scratch in
// PyTorch", Absorbing projections: attend directly to latents). For one query token the 128
// heads are the M = 128 rows of two dense contractions against the shared cache rows:
//   S = Q . K^T      (M = 128 heads, N = rows, K = 576 = [c_kv || k_rope])
//   O += P . V       (M = 128 heads, N = 512 latent dims, K = rows; V = the c_kv part of K)
//
// A tcgen05.mma instruction costs about the same whatever its N (up to 256), so both products
// are issued with N = 256: S over tiles of 256 rows (four 64-row cache blocks), O over 256
// latent dims at a time. O for 128 heads x 512 dims in fp32 fills one SM's tensor memory, so
// the two CTAs of a cluster take different roles for each work range:
//   * the score CTA keeps the latent part of Q in TMEM (256 columns, A operand) and its RoPE
//     part in shared memory, streams the cache rows' 64-dim slabs by TMA and accumulates S in
//     the other 256 TMEM columns. At each segment start Q's latent part comes through the same
//     TMA ring as the cache slabs and the MMA warp copies it into TMEM (tcgen05.cp), so a
//     switch to the next sequence costs the score CTA about one ring refill. Eight softmax warps copy S into registers (128 values per
//     thread) and release it at once, so the next tile's S = Q . K^T runs on the tensor core
//     while this tile's online softmax runs (exp2 units, O rescaled lazily only when the
//     running max grows by more than 2^8). P (bf16) and the per-row rescale factors and sums
//     go to the value CTA as 16 KB bulk copies into a 6-slot ring in its shared memory;
//   * the value CTA streams the latent part of the same rows by TMA and accumulates O = P . V
//     in its whole TMEM, applies rescales, and writes the normalised output.
// The two read the same cache blocks close together in time, so HBM sees each row about once.
// Warps of the score CTA: 0 TMA, 1 MMA issue, 2-9 softmax, 10 bulk copies to the value CTA.
// Warps of the value CTA: 0 TMA, 1 MMA issue, 2-5 rescale and epilogue, 6 acknowledgements to
// the score CTA (7-10 idle). No MMA-issuing warp ever waits on a cluster-scope fence.
// Every wait is bounded: on timeout the kernel sets MLA_DEV_WAIT_TIMEOUT, drains its copies
// and MMAs, frees TMEM and returns. No TMA multicast is used.
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_map.h"

namespace mla {
namespace {

constexpr int kH = 128;
constexpr int kR = 512;
constexpr int kDR = 64;
constexpr int kD = kR + kDR;
constexpr int kRows = 64;                       // rows per cache block = planner chunk
constexpr int kTileBlocks = 4;                  // blocks per score tile (N <= 256)
constexpr int kSlabBytes = kRows * 64 * 2;      // 64 rows x 64 dims bf16: 8 KB
constexpr int kThreads = 352;  // 11 warps
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait

// score CTA: K stages of one 64-dim slab for up to four blocks, RoPE part of Q, P staging
constexpr int kKStages = 4;
constexpr int kKStageBytes = kTileBlocks * kSlabBytes;        // 32 KB
constexpr int kQRopeBytes = kH * 64 * 2;                      // 16 KB
constexpr int kQBoxBytes = kH * 64 * 2;                       // 128 heads x 64 dims
constexpr int kQStages = kR / 128;                            // ring uses for Q's latent part
constexpr int kPBlockBytes = kH * kRows * 2;                  // 128 x 64 bf16: 16 KB
constexpr int kHdrBytes = 2 * kH * 4;                         // alpha[128], l[128]
constexpr int kS_K = 0;
constexpr int kS_QRope = kS_K + kKStages * kKStageBytes;      // 128 KB
constexpr int kS_Stage = kS_QRope + kQRopeBytes;              // 144 KB
constexpr int kS_Hdr = kS_Stage + kTileBlocks * kPBlockBytes; // 208 KB
constexpr int kS_Red = kS_Hdr + kHdrBytes;                    // row max / sum exchange
constexpr int kS_End = kS_Red + 4 * kH * 4;
// value CTA: V stages (one block's 256-dim half), P ring, header ring
constexpr int kVStages = 3;
constexpr int kVStageBytes = 4 * kSlabBytes;                  // 32 KB
constexpr int kPSlots = 6;
constexpr int kHdrSlots = 2;
constexpr int kV_V = 0;
constexpr int kV_P = kV_V + kVStages * kVStageBytes;          // 96 KB
constexpr int kV_Hdr = kV_P + kPSlots * kPBlockBytes;         // 192 KB
// output staging: per epilogue warp one 4 KB box of 32 rows x 32 fp32 (a TMA store source)
constexpr int kOutBoxBytes = 32 * 32 * 4;
constexpr int kV_Out = kV_Hdr + kHdrSlots * kHdrBytes;        // 194 KB (1 KB aligned)
constexpr int kV_End = kV_Out + 4 * kOutBoxBytes;
constexpr int kDataBytes = kS_End > kV_End ? kS_End : kV_End;

enum Bar {
  // score CTA
  kKFull = 0,
  kKEmpty = kKFull + kKStages,
  kQFull = kKEmpty + kKStages,  // RoPE part of the segment's Q in shared memory
  kQEmpty,                      // last S product of the segment done with Q
  kSFull,                       // S complete
  kSFree,                       // softmax done reading S
  kStgFree,                     // value CTA received the previous tile's P (staging reusable)
  kStaged,                      // softmax warps finished writing a tile's P and header
  kSlotFree,                    // kPSlots: value CTA finished with a P ring slot
  kRedMax = kSlotFree + kPSlots,  // the 8 softmax warps posted their row maxima
  kRedSum,                        // ... and their row sums
  // value CTA
  kVFull = kRedSum + 1,
  kVEmpty = kVFull + kVStages,
  kPFull = kVEmpty + kVStages,  // kPSlots
  kHFull = kPFull + kPSlots,    // kHdrSlots
  kSlotDone = kHFull + kHdrSlots,  // kPSlots: P . V MMAs reading a slot are complete
  kOReady = kSlotDone + kPSlots,   // rescale (if any) applied, previous epilogue done
  kPvDone,                         // 2: all P . V of a tile complete (even / odd tiles)
  kHdrRead = kPvDone + 2,          // the 4 epilogue warps have read a header slot
  kFinal,
  kNumBars
};
constexpr int kBarOff = kDataBytes;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // +1024: manual alignment

constexpr uint32_t kIdescPV = idesc(128, 256, 1);


struct Ctl {
  uint32_t* err;
  volatile int* abort;
};

// Warp-collective bounded wait; the result is the same in all 32 lanes. The first poll is
// inlined: with a call at every wait the kernel ran about 10% slower.
__device__ __noinline__ bool warp_wait_slow(uint32_t bar, uint32_t parity, const Ctl& c) {
  uint64_t t0 = 0;
  for (int it = 0;; ++it) {
    const bool done = mbar_try(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    if (it == 0) t0 = globaltimer();
    const bool late = (globaltimer() - t0) > kTimeoutNs;
    const bool stop = *c.abort != 0 || late;
    if (__any_sync(0xffffffffu, stop)) {
      if ((threadIdx.x & 31) == 0 && late) {
        set_error(c.err, MLA_DEV_WAIT_TIMEOUT);
        *c.abort = 1;
      }
      return false;
    }
  }
}
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  return warp_wait_slow(bar, parity, c);
}

// Barrier of a group of warps on an mbarrier that counts one arrival per warp: the k-th use
// (k = 0, 1, ...) waits for parity k & 1. Bounded like every other wait, so a warp that gave
// up elsewhere cannot leave the rest of its group blocked.
__device__ __forceinline__ bool group_sync(uint32_t bar, int k, const Ctl& c) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  return warp_wait(bar, (uint32_t)k & 1u, c);
}

// Bounded wait for a phase that normally completed long ago (drains at teardown).
__device__ void drain_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
  const uint64_t t0 = globaltimer();
  bool done = false;
  while (!done && globaltimer() - t0 < kTimeoutNs) done = __all_sync(0xffffffffu, mbar_try(bar, parity));
  if (!done && (threadIdx.x & 31) == 0) set_error(err, MLA_DEV_WAIT_TIMEOUT);
}

// One score tile: up to four consecutive cache blocks of one segment.
struct Tile {
  int bt, b, local0, nb, ntok, slot;
  bool first, last;
};

// Walks the tiles of segments [s, se) in order (identically in both CTAs).
struct TileWalk {
  const DecodeParams* p;
  int s, se, c;  // current segment and chunk
  __device__ bool next(Tile& tl) {
    while (s < se) {
      const Segment sg = p->segments[s];
      if (c < sg.chunk_lo) c = sg.chunk_lo;
      if (c < sg.chunk_hi) {
        const int chunk0 = p->bt_chunk0[sg.bt];
        tl.bt = sg.bt;
        tl.b = sg.bt / p->T;
        tl.local0 = c - chunk0;
        tl.nb = min(kTileBlocks, sg.chunk_hi - c);
        tl.ntok = min(tl.nb * kRows, p->bt_len[sg.bt] - tl.local0 * kRows);
        tl.slot = sg.slot;
        tl.first = (c == sg.chunk_lo);
        tl.last = (c + tl.nb == sg.chunk_hi);
        c += tl.nb;
        return true;
      }
      ++s;
      c = -1;
    }
    return false;
  }
};

// Block ids of a tile (lane j < nb holds block j), out-of-pool ids flagged and replaced by 0.
__device__ __forceinline__ int tile_block(const DecodeParams& p, const Tile& tl, int lane) {
  int blk = 0;
  if (lane < tl.nb) {
    blk = p.table[(size_t)tl.b * p.max_blocks + tl.local0 + lane];
    if (blk < 0 || blk >= p.num_blocks) {
      set_error(p.err, MLA_DEV_OOB_BLOCK);
      blk = 0;
    }
  }
  return blk;
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(168)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                 const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_out,
                 const __grid_constant__ CUtensorMap tm_part, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s_base = saddr(smem);
  const uint32_t s_bar = s_base + kBarOff;
  uint32_t* tmem_slot = (uint32_t*)(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = (volatile int*)(smem + kBarOff + kNumBars * 8 + 4);
  auto bar = [&](int i) { return s_bar + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const bool score = (rank == 0);
  const Ctl ctl{p.err, abort_flag};

  if (threadIdx.x == 0) {
    if (score) {
      for (int i = 0; i < kKStages; ++i) {
        mbar_init(bar(kKFull + i), 1);
        mbar_init(bar(kKEmpty + i), 1);
      }
      mbar_init(bar(kQFull), 1);
      mbar_init(bar(kQEmpty), 1);
      mbar_init(bar(kSFull), 1);
      mbar_init(bar(kSFree), 8);
      mbar_init(bar(kStgFree), 1);
      mbar_init(bar(kStaged), 8);
      for (int i = 0; i < kPSlots; ++i) mbar_init(bar(kSlotFree + i), 1);
      mbar_init(bar(kRedMax), 8);
      mbar_init(bar(kRedSum), 8);
    } else {
      for (int i = 0; i < kVStages; ++i) {
        mbar_init(bar(kVFull + i), 1);
        mbar_init(bar(kVEmpty + i), 1);
      }
      for (int i = 0; i < kPSlots; ++i) {
        mbar_init(bar(kPFull + i), 1);
        mbar_init(bar(kSlotDone + i), 1);
      }
      for (int i = 0; i < kHdrSlots; ++i) mbar_init(bar(kHFull + i), 1);
      mbar_init(bar(kOReady), 4);
      mbar_init(bar(kPvDone), 1);
      mbar_init(bar(kPvDone + 1), 1);
      mbar_init(bar(kHdrRead), 4);
      // every P slot and header slot expects one bulk copy from the score CTA per use
      for (int i = 0; i < kPSlots; ++i) mbar_expect_tx(bar(kPFull + i), kPBlockBytes);
      for (int i = 0; i < kHdrSlots; ++i) mbar_expect_tx(bar(kHFull + i), kHdrBytes);
    }
    mbar_init(bar(kFinal), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  cluster_sync();  // barriers of both CTAs initialised before any remote traffic
  const uint32_t tmem = *tmem_slot;
  wait_prior_grid();  // the schedule, Q and the cache rows come from earlier kernels

  const int q = blockIdx.x >> 1;
  int sb = 0, se = 0;
  if (q < p.header[1]) {
    sb = p.range_begin[q];
    se = p.range_begin[q + 1];
  }
  TileWalk walk{&p, sb, se, -1};
  Tile tl;

  if (score && warp == 0) {
    // ---------------------------------------------------------------- score: TMA producer
    int kt = 0, seg_i = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (tl.first) {
        // Q's latent part passes through the K ring (two 64-dim boxes of 128 heads per stage);
        // the MMA warp copies it into TMEM. The ring keeps streaming: these loads only wait
        // for stages that the previous segment's last products have released.
        for (int qs = 0; qs < kQStages && ok; ++qs, ++kt) {
          const int stage = kt % kKStages;
          if (kt >= kKStages &&
              !warp_wait(bar(kKEmpty + stage), ((kt / kKStages) - 1) & 1, ctl)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_expect_tx(bar(kKFull + stage), kKStageBytes);
            for (int b = 0; b < 2; ++b)
              tma_load(s_base + kS_K + stage * kKStageBytes + b * kQBoxBytes, &tm_q,
                       bar(kKFull + stage), 64 * (2 * qs + b), tl.bt * kH);
          }
          __syncwarp();
        }
        if (!ok) break;
        // RoPE part of Q into its own buffer, once the previous segment's S is done with it
        if (seg_i > 0 && !warp_wait(bar(kQEmpty), (seg_i - 1) & 1, ctl)) break;
        if (lane == 0) {
          mbar_expect_tx(bar(kQFull), kQRopeBytes);
          tma_load(s_base + kS_QRope, &tm_q, bar(kQFull), kR, tl.bt * kH);
        }
        __syncwarp();
        ++seg_i;
      }
      const int my_blk = tile_block(p, tl, lane);
      for (int k = 0; k < 9 && ok; ++k, ++kt) {  // 8 latent slabs, then the RoPE slab
        const int stage = kt % kKStages;
        if (kt >= kKStages && !warp_wait(bar(kKEmpty + stage), ((kt / kKStages) - 1) & 1, ctl)) {
          ok = false;
          break;
        }
#ifdef MLA_TEST_DROP_ARRIVE
        // test build only: the first work range never loads its sixth K slab, so the MMA
        // warp's bounded wait for it runs out and the kernel must report MLA_DEV_WAIT_TIMEOUT,
        // drain what it issued, free TMEM and return
        if (blockIdx.x < 2 && kt == 5) continue;
#endif
        if (lane == 0) mbar_expect_tx(bar(kKFull + stage), tl.nb * kSlabBytes);
        for (int j = 0; j < tl.nb; ++j) {
          const int blk = __shfl_sync(0xffffffffu, my_blk, j);
          if (lane == 0)
            tma_load(s_base + kS_K + stage * kKStageBytes + j * kSlabBytes, &tm_kv,
                     bar(kKFull + stage), 64 * k, blk * kRows);
        }
        __syncwarp();
      }
    }
    for (int k = 1; k <= kKStages && k <= kt; ++k)
      drain_wait(bar(kKFull + (kt - k) % kKStages), ((kt - k) / kKStages) & 1, p.err);
    if (seg_i > 0) drain_wait(bar(kQFull), (seg_i - 1) & 1, p.err);
  } else if (score && warp == 1) {
    // ---------------------------------------------------------------- score: S = Q . K^T
    int kt = 0, t = 0, seg_i = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (tl.first) {
        // the previous segment's S products have finished reading Q from TMEM
        if (seg_i > 0) ok = warp_wait(bar(kQEmpty), (seg_i - 1) & 1, ctl);
        // Q's latent part, staged by TMA in the K ring, into TMEM columns 256..511 (head h
        // in lane h, dims 2c and 2c + 1 in column 256 + c): 16 dims per copy, from the same
        // K-major 128-byte-swizzled layout an MMA operand descriptor reads. Copies and the
        // MMAs after them are issued by this thread and execute in order.
        for (int qs = 0; qs < kQStages && ok; ++qs, ++kt) {
          const int stage = kt % kKStages;
          if (!warp_wait(bar(kKFull + stage), (kt / kKStages) & 1, ctl)) {
            ok = false;
            break;
          }
          tc_after();
          if (lane == 0) {
            const uint32_t sb = s_base + kS_K + stage * kKStageBytes;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
              for (int i = 0; i < 4; ++i)
                tmem_cp128x256b(tmem + 256 + 32 * (2 * qs + b) + 8 * i,
                                sdesc(sb + b * kQBoxBytes + 32 * i, 16, 1024, 2));
            tc_commit(bar(kKEmpty + stage));
          }
          __syncwarp();
        }
        if (ok) ok = warp_wait(bar(kQFull), seg_i & 1, ctl);
        ++seg_i;
      }
      if (ok && t > 0) ok = warp_wait(bar(kSFree), (t - 1) & 1, ctl);
      if (!ok) break;
      const uint32_t id = idesc(128, kRows * tl.nb, 0);
#pragma unroll
      for (int k = 0; k < 9; ++k, ++kt) {
        const int stage = kt % kKStages;
        if (!warp_wait(bar(kKFull + stage), (kt / kKStages) & 1, ctl)) {
          ok = false;
          break;
        }
        tc_after();
        if (lane == 0) {
          const uint32_t kb = s_base + kS_K + stage * kKStageBytes;
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // 16 dims per step; B K-major, 8-row groups 1024 B apart
            const uint64_t bd = sdesc(kb + 32 * i, 16, 1024, 2);
            const uint32_t acc = (k > 0 || i > 0) ? 1u : 0u;
            if (k < 8)
              mma_ts(tmem, tmem + 256 + 32 * k + 8 * i, bd, id, acc);
            else
              mma_ss(tmem, sdesc(s_base + kS_QRope + 32 * i, 16, 1024, 2), bd, id, acc);
          }
          tc_commit(bar(kKEmpty + stage));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(bar(kSFull));
        if (tl.last) tc_commit(bar(kQEmpty));
      }
      __syncwarp();
      ++t;
    }
  } else if (score && warp >= 2 && warp < 10) {
    // ---------------------------------------------------------------- score: softmax, P staged
    // Eight warps: warp w reads TMEM lanes 32 * (w % 4) (its heads) and S columns
    // 128 * half .. +127 (two cache blocks). S is copied into registers at once and released,
    // so the MMA warp computes the next tile's S while this tile's softmax runs.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int h = quad * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;  // scores in log2 units
    const uint32_t stage_p = s_base + kS_Stage;
    const uint32_t hdr = s_base + kS_Hdr;
    float* red = (float*)(smem + kS_Red);  // [0..255]: max of half 0 / 1; [256..511]: sums

    int t = 0;
    float m_ref = 0.f, l = 0.f;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (!warp_wait(bar(kSFull), t & 1, ctl)) break;
      tc_after();
      uint32_t v[128];
      tmem_ld128(tq + 128 * half, v);
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kSFree));  // the next tile's S may be computed now
      // pass 1: row max over the valid rows of both halves
      const int lim = tl.ntok - 128 * half;
      float mt = -INFINITY;
#pragma unroll
      for (int k = 0; k < 128; ++k)
        if (k < lim) mt = fmaxf(mt, __uint_as_float(v[k]));
      red[half * kH + h] = mt;
      if (!group_sync(bar(kRedMax), t, ctl)) break;
      mt = fmaxf(red[h], red[kH + h]) * c2;
      float alpha = 1.f;
      if (tl.first) {
        m_ref = mt;
        l = 0.f;
      } else if (mt > m_ref + 8.f) {
        alpha = ex2(m_ref - mt);
        m_ref = mt;
      }
      // the value CTA must have received the previous tile before staging is overwritten
      if (t > 0 && !warp_wait(bar(kStgFree), (t - 1) & 1, ctl)) break;
      // pass 2: P = exp2(s * c2 - m_ref), rounded to bf16, packed in place, into the A-operand
      // layout of the value CTA's P . V (K-major, 128-byte rows swizzled by row % 8)
      float rs = 0.f;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const float p0 = (2 * k < lim) ? ex2(__uint_as_float(v[2 * k]) * c2 - m_ref) : 0.f;
        const float p1 = (2 * k + 1 < lim) ? ex2(__uint_as_float(v[2 * k + 1]) * c2 - m_ref) : 0.f;
        rs += p0;
        rs += p1;
        v[k] = pack_bf16(p0, p1);
      }
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const uint32_t row = stage_p + (2 * half + cb) * kPBlockBytes + (uint32_t)h * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           row + 16u * (uint32_t)(u ^ (h & 7))),
                       "r"(v[32 * cb + 4 * u]), "r"(v[32 * cb + 4 * u + 1]),
                       "r"(v[32 * cb + 4 * u + 2]), "r"(v[32 * cb + 4 * u + 3])
                       : "memory");
      }
      red[2 * kH + half * kH + h] = rs;
      if (!group_sync(bar(kRedSum), t, ctl)) break;
      if (half == 0) {
        rs += red[3 * kH + h];
        l = l * alpha + rs;
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(hdr + 4u * h), "f"(alpha) : "memory");
        if (tl.last) asm volatile("st.shared.f32 [%0], %1;" ::"r"(hdr + 4u * (kH + h)), "f"(l) : "memory");
      }
      fence_proxy_async();  // staged bytes are read by the bulk copies (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kStaged));
      if (tl.last && half == 0) {
        const float lse = (m_ref + __log2f(l)) * 0.6931471805599453f;
        if (tl.slot < 0) {
          if (p.lse) p.lse[(size_t)tl.bt * kH + h] = lse;
        } else {
          p.part_lse[(size_t)tl.slot * kH + h] = lse;
        }
      }
      ++t;
    }
  } else if (score && warp == 10) {
    // ---------------------------------------------------------------- score: ship P out
    const uint32_t peer_slots = peer_addr(s_base + kV_P, peer);
    const uint32_t peer_hdr = peer_addr(s_base + kV_Hdr, peer);
    int t = 0, g = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      ok = warp_wait(bar(kStaged), t & 1, ctl);
      for (int c = 0; c < tl.nb && ok; ++c) {  // the ring slot's previous block is done
        const int gb = g + c;
        if (gb >= kPSlots)
          ok = warp_wait(bar(kSlotFree + gb % kPSlots), ((gb / kPSlots) - 1) & 1, ctl);
      }
      if (!ok) break;
      if (lane == 0) {
        const int hs = t % kHdrSlots;
        bulk_to_peer(peer_hdr + hs * kHdrBytes, s_base + kS_Hdr, kHdrBytes,
                     peer_addr(bar(kHFull + hs), peer));
        for (int c = 0; c < tl.nb; ++c) {
          const int slot = (g + c) % kPSlots;
          bulk_to_peer(peer_slots + slot * kPBlockBytes, s_base + kS_Stage + c * kPBlockBytes,
                       kPBlockBytes, peer_addr(bar(kPFull + slot), peer));
        }
      }
      __syncwarp();
      g += tl.nb;
      ++t;
    }
  } else if (!score && warp == 6) {
    // ---------------------------------------------------------------- value: acknowledgements
    int t = 0, g = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      // the whole tile arrived: the score CTA may overwrite its staging
      for (int j = 0; j < tl.nb && ok; ++j)
        ok = warp_wait(bar(kPFull + (g + j) % kPSlots), ((g + j) / kPSlots) & 1, ctl);
      if (ok) ok = warp_wait(bar(kHFull + t % kHdrSlots), (t / kHdrSlots) & 1, ctl);
      if (!ok) break;
      if (lane == 0) mbar_arrive_peer(peer_addr(bar(kStgFree), peer));
      __syncwarp();
      // each ring slot is free once the P . V that read it completed
      for (int j = 0; j < tl.nb && ok; ++j, ++g) {
        ok = warp_wait(bar(kSlotDone + g % kPSlots), (g / kPSlots) & 1, ctl);
        if (ok && lane == 0) mbar_arrive_peer(peer_addr(bar(kSlotFree + g % kPSlots), peer));
        __syncwarp();
      }
      ++t;
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- value: TMA producer
    // This is the second and last read of these lines: evict them first, so that L2 keeps
    // the score CTA's fresh loads, the partial outputs and the projection weights instead.
    const uint64_t pol_drop = l2_evict_first();
    int vt = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      const int my_blk = tile_block(p, tl, lane);
      for (int j = 0; j < tl.nb && ok; ++j) {
        const int blk = __shfl_sync(0xffffffffu, my_blk, j);
        for (int dh = 0; dh < 2; ++dh, ++vt) {
          const int vs = vt % kVStages;
          if (vt >= kVStages && !warp_wait(bar(kVEmpty + vs), ((vt / kVStages) - 1) & 1, ctl)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_expect_tx(bar(kVFull + vs), kVStageBytes);
            for (int i = 0; i < 4; ++i)
              tma_load_hint(s_base + kV_V + vs * kVStageBytes + i * kSlabBytes, &tm_kv,
                            bar(kVFull + vs), 256 * dh + 64 * i, blk * kRows, pol_drop);
          }
          __syncwarp();
        }
      }
    }
    for (int k = 1; k <= kVStages && k <= vt; ++k)
      drain_wait(bar(kVFull + (vt - k) % kVStages), ((vt - k) / kVStages) & 1, p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- value: O += P . V
    int vt = 0, g = 0, t = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      // the whole tile's P and header arrived: the score CTA may reuse its staging
      for (int j = 0; j < tl.nb && ok; ++j)
        ok = warp_wait(bar(kPFull + (g + j) % kPSlots), ((g + j) / kPSlots) & 1, ctl);
      if (ok) ok = warp_wait(bar(kHFull + t % kHdrSlots), (t / kHdrSlots) & 1, ctl);
      if (ok) ok = warp_wait(bar(kOReady), t & 1, ctl);
      if (!ok) break;
      if (lane == 0)
        for (int j = 0; j < tl.nb; ++j)  // re-arm for each slot's next use
          mbar_expect_tx(bar(kPFull + (g + j) % kPSlots), kPBlockBytes);
      __syncwarp();
      for (int j = 0; j < tl.nb && ok; ++j, ++g) {
        const int slot = g % kPSlots;
        const int valid = min(kRows, tl.ntok - kRows * j);
        for (int dh = 0; dh < 2; ++dh, ++vt) {
          const int vs = vt % kVStages;
          if (!warp_wait(bar(kVFull + vs), (vt / kVStages) & 1, ctl)) {
            ok = false;
            break;
          }
          if (valid < kRows) {
            // rows past the sequence end: zero them so 0 * garbage never enters P . V
            uint8_t* st = smem + kV_V + vs * kVStageBytes;
            const int n16 = (kRows - valid) * 128 / 16;
            for (int slab = 0; slab < 4; ++slab) {
              uint4* z = (uint4*)(st + slab * kSlabBytes + valid * 128);
              for (int i = lane; i < n16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();
            __syncwarp();
          }
          tc_after();
          if (lane == 0) {
            const uint32_t vb = s_base + kV_V + vs * kVStageBytes;
            const uint32_t pb = s_base + kV_P + slot * kPBlockBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i)  // 16 rows per step; B MN-major: LBO = 64-dim slab
              mma_ss(tmem + 256 * dh, sdesc(pb + 32 * i, 16, 1024, 2),
                     sdesc(vb + 2048 * i, kSlabBytes, 1024, 2), kIdescPV,
                     (tl.first && j == 0 && i == 0) ? 0u : 1u);
            tc_commit(bar(kVEmpty + vs));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit(bar(kSlotDone + slot));
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar(kPvDone + (t & 1)));
      __syncwarp();
      ++t;
    }
  } else if (!score && warp >= 2 && warp < 6) {
    // ---------------------------------------------------------------- value: rescale, epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    int t = 0;
    float l_last = 1.f;
    bool ok = true;
    // Completions of P . V are observed tile by tile, in order: a parity wait is only
    // unambiguous when the phase before it has been seen. Tile k's phase on barrier k & 1 can
    // only be followed by tile k + 2's, which needs this warp's OReady of tile k + 2 first.
    int pv_next = 0;
    auto wait_pv = [&](int k) -> bool {
      while (pv_next <= k) {
        if (!warp_wait(bar(kPvDone + (pv_next & 1)), (pv_next >> 1) & 1, ctl)) return false;
        ++pv_next;
      }
      return true;
    };
    while (ok && walk.next(tl)) {
      const int hs = t % kHdrSlots;
      if (!warp_wait(bar(kHFull + hs), (t / kHdrSlots) & 1, ctl)) break;
      const uint32_t hb = s_base + kV_Hdr + hs * kHdrBytes;
      float alpha;
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(alpha) : "r"(hb + 4u * h) : "memory");
      if (tl.last) asm volatile("ld.shared.f32 %0, [%1];" : "=f"(l_last) : "r"(hb + 4u * (kH + h)) : "memory");
      if (!group_sync(bar(kHdrRead), t, ctl)) break;  // all read it before it is re-armed
      if (threadIdx.x == 64) mbar_expect_tx(bar(kHFull + hs), kHdrBytes);
      if (!tl.first && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_pv(t - 1)) break;
        tc_after();
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
          uint32_t o[32];
          tmem_ld32(tq + 32 * ch, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tq + 32 * ch, o);
        }
        tmem_wait_st();
      }
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOReady));
      if (!tl.last) {
        if (t > 0 && !wait_pv(t - 1)) break;  // keep up with completions
      } else {
        if (!wait_pv(t)) break;
        tc_after();
        const float inv_l = 1.f / l_last;
        // O / l leaves through shared memory: each warp stages its 32 rows x 32 columns as a
        // 128-byte-swizzled 4 KB box and one lane stores the box with TMA, so the global
        // writes are whole lines rather than 16-byte pieces 2 KB apart.
        // kept in L2: the combine (partials) and the output projection (O) read them next,
        // after the rest of the cache has streamed through
        const uint64_t keep = l2_evict_last();
        const CUtensorMap* map = tl.slot < 0 ? &tm_out : &tm_part;
        const int row0 = (tl.slot < 0 ? tl.bt : tl.slot) * kH + quad * 32;
        const uint32_t box = s_base + kV_Out + (uint32_t)quad * kOutBoxBytes;
        // the next chunk's TMEM load is in flight while this chunk is staged and stored
        uint32_t o[32], nx[32];
        tmem_ld32(tq, o);
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
          if (ch + 1 < 16) tmem_ld32_async(tq + 32 * (ch + 1), nx);
          if (ch >= 1) {  // the previous chunk's store is done reading the box
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
          }
          const uint32_t row = box + (uint32_t)lane * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                             row + 16u * (uint32_t)(u ^ (lane & 7))),
                         "f"(__uint_as_float(o[4 * u]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 1]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 2]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 3]) * inv_l)
                         : "memory");
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) tma_store_hint(map, box, 32 * ch, row0, keep);
          if (ch + 1 < 16) {
            tmem_wait_ld(nx);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = nx[i];
          }
        }
        if (lane == 0) bulk_wait_read<0>();  // the box is free for the next segment
        __syncwarp();
        tc_before();
      }
      ++t;
    }
  }

  // ---------------------------------------------------------------------- teardown
  if (!score && warp >= 2 && warp < 6 && lane == 0) bulk_wait_all();  // output stores landed
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 1) {
    if (lane == 0) tc_commit(bar(kFinal));  // completes once every MMA issued here is done
    __syncwarp();
    drain_wait(bar(kFinal), 0, p.err);
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
  cluster_sync();  // the peer no longer touches this CTA's shared memory
}

bool tc_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.num_heads == kH && c.kv_rank == kR && c.rope_dim == kDR &&
         c.block_size == kRows;
}

cudaError_t launch_attend_tc(const mla_config& c, const DecodeParams& p, cudaStream_t st) {
  (void)c;
  CUtensorMap kv, qm, om, pm;
  if (!make_bf16_map(&kv, p.pool, kD, (uint64_t)p.num_blocks * kRows, kD * 2, kRows) ||
      !make_bf16_map(&qm, p.q, kD, (uint64_t)p.BT * kH, kD * 2, kH) ||
      !make_f32_box32_map(&om, p.out, kR, (uint64_t)p.BT * kH) ||
      !make_f32_box32_map(&pm, p.part_o, kR, (uint64_t)kMaxPartials * kH))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(attend_tc_kernel, dim3(2 * kRanges), dim3(kThreads), kSmemBytes, st, kv, qm,
                    om, pm, p);
}

}  // namespace mla
