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
// A tcgen05.mma of M = 128, K = 16 costs N / 2 cycles, but its issue blocks the issuing thread
// until it is about to run, and every mbarrier read in that thread costs more than an N = 128
// MMA takes: only N = 256 MMAs keep the tensor pipe busy across the per-stage barrier waits. So
// both products are issued with N = 256: S over tiles of 256 rows (four 64-row cache blocks), O
// over 256 latent dims at a time. O for 128 heads x 512 dims in fp32 fills one SM's tensor
// memory, so the two CTAs of a cluster take different roles for each work range:
//   * the score CTA keeps the latent part of Q in TMEM (256 columns, A operand) and its RoPE
//     part in shared memory, streams the cache rows' 64-dim slabs by TMA (a 4-stage ring of
//     32 KB stages) and accumulates S in the other 256 TMEM columns. At each segment start Q's
//     latent part comes through the same ring and the MMA warp copies it into TMEM
//     (tcgen05.cp). Eight softmax warps copy S into registers (a thread: one head, 128 rows)
//     and release it at once, so the next tile's S = Q . K^T runs on the tensor core while this
//     tile's softmax runs (exp2 units; the running maximum moves only when a tile's maximum
//     exceeds it by more than 2^8). P (bf16, in the A-operand layout of P . V) is computed in
//     registers before the staging buffer is free, then stored; P and the tile's header
//     (per-head rescale factor, and at a segment's end the final maximum) go to the value CTA
//     as bulk copies into a 4-slot ring in its shared memory, each block as soon as its slot
//     is free;
//   * the value CTA streams the latent part of the same rows by TMA and accumulates O = P . V
//     in its whole TMEM, sums each head's P row (the bf16 values the MMA consumes) into l,
//     applies rescales, and writes O / l and the log-sum-exp.
// The two read the same cache blocks close together in time, so HBM sees each row about once.
// Warps of the score CTA: 0 TMA, 1 MMA issue, 2-9 softmax (two per lane quarter, one per half
// of the tile's rows), 10 bulk copies to the value CTA. Warps of the value CTA: 0 TMA, 1 MMA
// issue, 2-5 row sums, rescale and epilogue, 6 acknowledgements to the score CTA (7-10 idle).
// Every wait is bounded: on timeout the kernel sets MLA_DEV_WAIT_TIMEOUT, drains its copies
// and MMAs (including bulk copies the peer has issued into its shared memory), frees TMEM and
// returns. No TMA multicast is used.
#include <atomic>

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
constexpr int kTileRows = kTileBlocks * kRows;  // 256
constexpr int kSlabBytes = kRows * 64 * 2;      // 64 rows x 64 dims bf16: 8 KB
constexpr int kThreads = 352;                   // 11 warps
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait

// score CTA: K stages of one 64-dim slab for up to four blocks, RoPE part of Q, P staging,
// header staging, row-maximum exchange between the two warps of a lane quarter
constexpr int kKStages = 4;
constexpr int kKStageBytes = kTileBlocks * kSlabBytes;        // 32 KB
constexpr int kQBoxBytes = kH * 64 * 2;                       // 128 heads x 64 dims: 16 KB
constexpr int kQStages = kR / 128;                            // ring uses for Q's latent part
static_assert(2 * kQBoxBytes == kKStageBytes, "two Q boxes fill one K stage");
constexpr int kQRopeBytes = kH * 64 * 2;                      // 16 KB
constexpr int kPBlockBytes = kH * kRows * 2;                  // 128 x 64 bf16: 16 KB
constexpr int kTilePBytes = kTileBlocks * kPBlockBytes;       // 64 KB
constexpr int kHdrBytes = 2 * kH * 4;                         // alpha[128], m_last[128]
constexpr int kS_K = 0;
constexpr int kS_QRope = kS_K + kKStages * kKStageBytes;      // 128 KB
constexpr int kS_Stage = kS_QRope + kQRopeBytes;              // 144 KB
constexpr int kS_Hdr = kS_Stage + kTilePBytes;                // 208 KB
constexpr int kS_Red = kS_Hdr + kHdrBytes;                    // 209 KB: max[2 tiles][2 halves][128]
constexpr int kS_End = kS_Red + 4 * kH * 4;
// value CTA: V stages (one block's 256-dim half), P ring (each slot: a P block + the header)
constexpr int kVStages = 4;
constexpr int kVStageBytes = 4 * kSlabBytes;                  // 32 KB
constexpr int kPSlots = 4;
constexpr int kSlotBytes = kPBlockBytes + kHdrBytes;          // 17 KB (1 KB aligned)
constexpr int kV_V = 0;
constexpr int kV_P = kV_V + kVStages * kVStageBytes;          // 128 KB
// output staging: per epilogue warp one 4 KB box of 32 rows x 32 fp32 (a transpose buffer)
constexpr int kOutBoxBytes = 32 * 32 * 4;
constexpr int kV_Out = kV_P + kPSlots * kSlotBytes;           // 196 KB (1 KB aligned)
constexpr int kV_End = kV_Out + 4 * kOutBoxBytes;             // 212 KB
constexpr int kDataBytes = kS_End > kV_End ? kS_End : kV_End;
// segments of the work range, staged once per CTA (longer ranges read the rest from global)
constexpr int kSegCache = 64;
constexpr int kSegOff = kDataBytes;
constexpr int kSegBytes = kSegCache * 28;

enum Bar {
  // score CTA
  kKFull = 0,
  kKEmpty = kKFull + kKStages,
  kQFull = kKEmpty + kKStages,  // RoPE part of the segment's Q in shared memory
  kQEmpty,                      // last S product of the segment done with Q
  kSFull,                       // S complete
  kSFree,                       // the eight softmax warps copied S out
  kStgFree,                     // value CTA received the previous tile (staging reusable)
  kStaged,                      // the eight softmax warps wrote the tile's P and header
  kSlotFree,                    // kPSlots: value CTA finished with a P ring slot
  kRed = kSlotFree + kPSlots,   // 4: the two warps of a lane quarter posted their row maxima
  // value CTA
  kVFull = kRed + 4,
  kVEmpty = kVFull + kVStages,
  kPFull = kVEmpty + kVStages,     // kPSlots: P block and header landed (armed at each use)
  kSlotDone = kPFull + kPSlots,    // kPSlots: P . V MMAs reading a slot are complete
  kOReady = kSlotDone + kPSlots,   // rescale (if any) applied, previous epilogue done
  kSumDone,                        // kPSlots: the four sum warps read a slot's P rows
  kPvDone = kSumDone + kPSlots,    // 2: all P . V of a tile complete (even / odd tiles)
  kFinal = kPvDone + 2,
  kNumBars
};
constexpr int kBarOff = kSegOff + kSegBytes;
// + tmem slot, abort flag, count of P blocks the score CTA sent (written into the value CTA)
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // +1024: manual alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

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

// Single-thread bounded wait, for loops that one lane runs alone (the MMA issue loops: a
// warp-wide poll and __syncwarp per stage cost more than four N = 128 MMAs take to execute).
__device__ __noinline__ bool thread_wait_slow(uint32_t bar, uint32_t parity, const Ctl& c) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (*c.abort != 0) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      set_error(c.err, MLA_DEV_WAIT_TIMEOUT);
      *c.abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool thread_wait(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try(bar, parity)) return true;
  return thread_wait_slow(bar, parity, c);
}

// Bounded wait for a phase that normally completed long ago (drains at teardown).
__device__ void drain_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
  const uint64_t t0 = globaltimer();
  bool done = false;
  while (!done && globaltimer() - t0 < kTimeoutNs) done = __all_sync(0xffffffffu, mbar_try(bar, parity));
  if (!done && (threadIdx.x & 31) == 0) set_error(err, MLA_DEV_WAIT_TIMEOUT);
}

// A segment of the work range with the fields of its row group (b: its sequence).
struct SegInfo {
  int bt, chunk_lo, chunk_hi, slot, chunk0, len, b;
};

__device__ __forceinline__ SegInfo load_segment(const DecodeParams& p, int s) {
  const Segment sg = p.segments[s];
  return SegInfo{sg.bt, sg.chunk_lo, sg.chunk_hi, sg.slot, p.bt_chunk0[sg.bt], p.bt_len[sg.bt],
                 sg.bt / p.T};
}

// One score tile: up to two consecutive cache blocks of one segment.
struct Tile {
  int bt, b, local0, nb, ntok, slot;
  bool first, last;
};

// Walks the tiles of segments [s, se) in order (identically in every warp of both CTAs). The
// current segment's fields are held in registers; they come from the CTA's shared-memory copy
// of the range's first kSegCache segments, or from global memory after those.
struct TileWalk {
  const DecodeParams* p;
  const SegInfo* cache;  // shared memory, segments sb .. sb + kSegCache - 1
  int sb, s, se, c;      // first segment of the range, current segment and chunk
  int loaded;            // index of the segment held in cur, or -1
  SegInfo cur;
  __device__ bool next(Tile& tl) {
    while (s < se) {
      if (loaded != s) {
        cur = (s - sb < kSegCache) ? cache[s - sb] : load_segment(*p, s);
        loaded = s;
      }
      if (c < cur.chunk_lo) c = cur.chunk_lo;
      if (c < cur.chunk_hi) {
        tl.bt = cur.bt;
        tl.b = cur.b;
        tl.local0 = c - cur.chunk0;
        tl.nb = min(kTileBlocks, cur.chunk_hi - c);
        tl.ntok = min(tl.nb * kRows, cur.len - tl.local0 * kRows);
        tl.slot = cur.slot;
        tl.first = (c == cur.chunk_lo);
        tl.last = (c + tl.nb == cur.chunk_hi);
        c += tl.nb;
        return true;
      }
      ++s;
      c = -1;
    }
    return false;
  }
};

// Block ids of a sequence read 32 table entries at a time: lane i holds the entry of chunk
// base + i. Out-of-pool ids are flagged at use and replaced by 0.
struct BlockWindow {
  int b = -1, base = 0, blk = 0;
  __device__ int get(const DecodeParams& p, int seq, int local, int lane) {
    if (seq != b || local < base || local >= base + 32) {  // warp-uniform
      b = seq;
      base = local;
      const int chunk = local + lane;
      blk = chunk < p.max_blocks ? p.table[(size_t)seq * p.max_blocks + chunk] : 0;
    }
    int id = __shfl_sync(0xffffffffu, blk, local - base);
    if (id < 0 || id >= p.num_blocks) {
      if (lane == 0) set_error(p.err, MLA_DEV_OOB_BLOCK);
      id = 0;
    }
    return id;
  }
};

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(168)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                 const __grid_constant__ CUtensorMap tm_q, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s_base = saddr(smem);
  const uint32_t s_bar = s_base + kBarOff;
  uint32_t* tmem_slot = (uint32_t*)(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = (volatile int*)(smem + kBarOff + kNumBars * 8 + 4);
  // value CTA: number of P blocks the score CTA sent (written remotely before the last sync)
  volatile int* sent_count = (volatile int*)(smem + kBarOff + kNumBars * 8 + 8);
  SegInfo* seg_cache = (SegInfo*)(smem + kSegOff);
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
      for (int i = 0; i < 4; ++i) mbar_init(bar(kRed + i), 2);
    } else {
      for (int i = 0; i < kVStages; ++i) {
        mbar_init(bar(kVFull + i), 1);
        mbar_init(bar(kVEmpty + i), 1);
      }
      for (int i = 0; i < kPSlots; ++i) {
        mbar_init(bar(kPFull + i), 1);
        mbar_init(bar(kSlotDone + i), 1);
      }
      mbar_init(bar(kOReady), 4);
      for (int i = 0; i < kPSlots; ++i) mbar_init(bar(kSumDone + i), 4);
      mbar_init(bar(kPvDone), 1);
      mbar_init(bar(kPvDone + 1), 1);
    }
    mbar_init(bar(kFinal), 1);
    *abort_flag = 0;
    *sent_count = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  wait_prior_grid();  // the schedule, Q and the cache rows come from earlier kernels

  const int q = blockIdx.x >> 1;
  int sb = 0, se = 0;
  if (q < p.header[1]) {
    sb = p.range_begin[q];
    se = p.range_begin[q + 1];
  }
  for (int i = threadIdx.x; i < min(se - sb, kSegCache); i += blockDim.x)
    seg_cache[i] = load_segment(p, sb + i);
  tc_before();
  __syncthreads();
  tc_after();
  cluster_sync();  // barriers of both CTAs initialised before any remote traffic
  const uint32_t tmem = *tmem_slot;

  TileWalk walk{&p, seg_cache, sb, sb, se, -1, -1, {}};
  Tile tl;
  int value_sent = 0;  // score CTA, warp 10: P blocks sent to the value CTA

  if (score && warp == 0) {
    // ---------------------------------------------------------------- score: TMA producer
    BlockWindow win;
    int kt = 0, seg_i = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (tl.first) {
        // Q's latent part passes through the K ring (two 64-dim boxes of 128 heads per stage);
        // the MMA warp copies it into TMEM. These loads only wait for stages that the
        // previous segment's last products have released.
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
      int blk[kTileBlocks];
#pragma unroll
      for (int j = 0; j < kTileBlocks; ++j)
        blk[j] = j < tl.nb ? win.get(p, tl.b, tl.local0 + j, lane) : 0;
      for (int k = 0; k < 9 && ok; ++k, ++kt) {  // 8 latent slabs, then the RoPE slab
        const int stage = kt % kKStages;
        if (kt >= kKStages && !warp_wait(bar(kKEmpty + stage), ((kt / kKStages) - 1) & 1, ctl)) {
          ok = false;
          break;
        }
#ifdef MLA_TEST_DROP_ARRIVE
        // test build only: the first work range never loads one K slab, so the MMA warp's
        // bounded wait for it runs out and the kernel must report MLA_DEV_WAIT_TIMEOUT, drain
        // what it issued, free TMEM and return
        if (blockIdx.x < 2 && kt == 9) continue;
#endif
        if (lane == 0) {
          mbar_expect_tx(bar(kKFull + stage), tl.nb * kSlabBytes);
#pragma unroll
          for (int j = 0; j < kTileBlocks; ++j)
            if (j < tl.nb)
              tma_load(s_base + kS_K + stage * kKStageBytes + j * kSlabBytes, &tm_kv,
                       bar(kKFull + stage), 64 * k, blk[j] * kRows);
        }
        __syncwarp();
      }
    }
    for (int k = 1; k <= kKStages && k <= kt; ++k)
      drain_wait(bar(kKFull + (kt - k) % kKStages), ((kt - k) / kKStages) & 1, p.err);
    if (seg_i > 0) drain_wait(bar(kQFull), (seg_i - 1) & 1, p.err);
  } else if (score && warp == 1) {
    // ---------------------------------------------------------------- score: S = Q . K^T
    // One lane runs the whole loop (a stage's barrier wait hides behind the N = 256 MMAs
    // still queued).
    if (lane == 0) {
      int kt = 0, t = 0, seg_i = 0;
      bool ok = true, next_ready = false;
      while (ok && walk.next(tl)) {
        if (tl.first) {
          // the previous segment's S products have finished reading Q from TMEM
          if (seg_i > 0) ok = thread_wait(bar(kQEmpty), (seg_i - 1) & 1, ctl);
          // Q's latent part, staged by TMA in the K ring, into TMEM columns 256..511 (head h
          // in lane h, dims 2c and 2c + 1 in column 256 + c): 16 dims per copy, from the same
          // K-major 128-byte-swizzled layout an MMA operand descriptor reads. Copies and the
          // MMAs after them are issued by this thread and execute in order.
          for (int qs = 0; qs < kQStages && ok; ++qs, ++kt) {
            const int stage = kt % kKStages;
            if (!thread_wait(bar(kKFull + stage), (kt / kKStages) & 1, ctl)) {
              ok = false;
              break;
            }
            tc_after();
            const uint32_t sb_ = s_base + kS_K + stage * kKStageBytes;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
              for (int i = 0; i < 4; ++i)
                tmem_cp128x256b(tmem + 256 + 32 * (2 * qs + b) + 8 * i,
                                sdesc(sb_ + b * kQBoxBytes + 32 * i, 16, 1024, 2));
            tc_commit(bar(kKEmpty + stage));
          }
          if (ok) ok = thread_wait(bar(kQFull), seg_i & 1, ctl);
          ++seg_i;
        }
        // S was copied out by the softmax of the previous tile
        if (ok && t >= 1) ok = thread_wait(bar(kSFree), (t - 1) & 1, ctl);
        if (!ok) break;
        const uint32_t id = idesc(128, kRows * tl.nb, 0);
        const uint32_t d = tmem;
        // a rolled loop: the issuing thread's code stays small, so that its instruction fetch
        // does not miss behind the softmax warps' unrolled code on the same scheduler. The
        // next stage's barrier is tested (without blocking) between a stage's MMAs, while two of
        // them are queued: a barrier read takes longer than one MMA, and a stage already seen
        // complete needs no wait at its start.
        if (tl.first) next_ready = false;
#pragma unroll 1
        for (int k = 0; k < 9; ++k, ++kt) {
          const int stage = kt % kKStages;
          if (!next_ready && !thread_wait(bar(kKFull + stage), (kt / kKStages) & 1, ctl)) {
            ok = false;
            break;
          }
          tc_after();
          const uint32_t kb = s_base + kS_K + stage * kKStageBytes;
          const int nkt = kt + 1;
          if (k < 8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // 16 dims per step; B K-major, 8-row groups 1024 B apart
              mma_ts(d, tmem + 256 + 32 * k + 8 * i, sdesc(kb + 32 * i, 16, 1024, 2), id,
                     (k > 0 || i > 0) ? 1u : 0u);
              if (i == 1) next_ready = mbar_test(bar(kKFull + nkt % kKStages), (nkt / kKStages) & 1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              mma_ss(d, sdesc(s_base + kS_QRope + 32 * i, 16, 1024, 2),
                     sdesc(kb + 32 * i, 16, 1024, 2), id, 1u);
              // the next tile's first stage (of the same segment; a new segment's first
              // stages carry its query and are waited for as usual)
              if (i == 1) next_ready = mbar_test(bar(kKFull + nkt % kKStages), (nkt / kKStages) & 1);
            }
          }
          tc_commit(bar(kKEmpty + stage));
        }
        if (!ok) break;
        tc_commit(bar(kSFull));
        if (tl.last) tc_commit(bar(kQEmpty));
        ++t;
      }
    }
    __syncwarp();
  } else if (score && warp >= 2 && warp < 10) {
    // ---------------------------------------------------------------- score: softmax, P staged
    // Eight warps: warp w reads TMEM lanes 32 * (w % 4) (its heads) and S columns
    // 128 * half .. +127 (two cache blocks). S is copied into registers at once and released,
    // so the MMA warp computes the next tile's S while this tile's softmax runs. The two warps
    // of a lane quarter exchange their half-tile maxima through shared memory (one buffer per
    // tile parity) and both keep the same running maximum m_ref.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int h = quad * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + 128u * (uint32_t)half;
    const float c2 = p.scale * 1.4426950408889634f;  // scores in log2 units
    float* red = (float*)(smem + kS_Red);            // [tile parity][half][head]
    const uint32_t stage_p = s_base + kS_Stage + (uint32_t)(2 * half) * kPBlockBytes;
    const uint32_t hdr = s_base + kS_Hdr;

    int t = 0;
    float m_ref = 0.f;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (!warp_wait(bar(kSFull), t & 1, ctl)) break;
      tc_after();
      uint32_t v[128];
      tmem_ld128(tq, v);
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kSFree));  // the next tile's S may be computed now
      // rows past the segment's end (stale or unwritten TMEM columns) count as -inf, which
      // drops them from the maximum and gives them P = exp2(-inf) = 0
      const int lim = tl.ntok - 128 * half;
      if (lim < 128) {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= lim) v[k] = 0xff800000u;
      }
      // pass 1: row max over this half (four independent chains of three-input max)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int k = 0; k < 128; k += 8)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          mx[c] = fmax3(mx[c], __uint_as_float(v[k + 2 * c]), __uint_as_float(v[k + 2 * c + 1]));
      float* rt = red + (t & 1) * 2 * kH;
      rt[half * kH + h] = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kRed + quad));
      if (!warp_wait(bar(kRed + quad), t & 1, ctl)) break;
      const float mt = fmaxf(rt[h], rt[kH + h]) * c2;
      float alpha = 1.f;
      if (tl.first) {
        m_ref = mt;
      } else if (mt > m_ref + 8.f) {
        alpha = ex2(m_ref - mt);
        m_ref = mt;
      }
      // pass 2 in registers: P = exp2(s * c2 - m_ref) (the argument two at a time, one packed
      // fma), rounded to bf16, packed in place
      const float2 c2x2 = make_float2(c2, c2), nm = make_float2(-m_ref, -m_ref);
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const float2 x = __ffma2_rn(
            make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])), c2x2, nm);
        v[k] = pack_bf16(ex2(x.x), ex2(x.y));
      }
      // the value CTA received the previous tile: the staging buffer may be overwritten
      if (t > 0 && !warp_wait(bar(kStgFree), (t - 1) & 1, ctl)) break;
      if (half == 0) {
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(hdr + 4u * h), "f"(alpha) : "memory");
        if (tl.last)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(hdr + 4u * (kH + h)), "f"(m_ref) : "memory");
      }
      // P into the A-operand layout of the value CTA's P . V (K-major, 128-byte rows swizzled
      // by row % 8), blocks 2 * half and 2 * half + 1
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const uint32_t row = stage_p + cb * kPBlockBytes + (uint32_t)h * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           row + 16u * (uint32_t)(u ^ (h & 7))),
                       "r"(v[32 * cb + 4 * u]), "r"(v[32 * cb + 4 * u + 1]),
                       "r"(v[32 * cb + 4 * u + 2]), "r"(v[32 * cb + 4 * u + 3])
                       : "memory");
      }
      fence_proxy_async();  // staged bytes are read by the bulk copies (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kStaged));
      ++t;
    }
  } else if (score && warp == 10) {
    // ---------------------------------------------------------------- score: ship P out
    // Every block goes to its own ring slot together with the tile's header (the value CTA
    // reads the header of a tile's first block).
    const uint32_t peer_slots = peer_addr(s_base + kV_P, peer);
    int t = 0, g = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      ok = warp_wait(bar(kStaged), t & 1, ctl);
      for (int c = 0; c < tl.nb && ok; ++c) {
        const int gb = g + c;
        // the ring slot's previous block is done; then this block goes at once
        if (gb >= kPSlots)
          ok = warp_wait(bar(kSlotFree + gb % kPSlots), ((gb / kPSlots) - 1) & 1, ctl);
        if (!ok) break;
        if (lane == 0) {
          const int slot = gb % kPSlots;
          const uint32_t dst = peer_slots + slot * kSlotBytes;
          const uint32_t pbar = peer_addr(bar(kPFull + slot), peer);
          bulk_to_peer(dst, s_base + kS_Stage + c * kPBlockBytes, kPBlockBytes, pbar);
          bulk_to_peer(dst + kPBlockBytes, s_base + kS_Hdr, kHdrBytes, pbar);
        }
        __syncwarp();
        ++value_sent;
      }
      if (!ok) break;
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
      if (!ok) break;
      if (lane == 0) mbar_arrive_peer(peer_addr(bar(kStgFree), peer));
      __syncwarp();
      // each ring slot is free once the P . V that read it completed and its row sums are done
      for (int j = 0; j < tl.nb && ok; ++j) {
        const int gb = g + j;
        ok = warp_wait(bar(kSlotDone + gb % kPSlots), (gb / kPSlots) & 1, ctl) &&
             warp_wait(bar(kSumDone + gb % kPSlots), (gb / kPSlots) & 1, ctl);
        if (ok && lane == 0) mbar_arrive_peer(peer_addr(bar(kSlotFree + gb % kPSlots), peer));
        __syncwarp();
      }
      if (!ok) break;
      g += tl.nb;
      ++t;
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- value: TMA producer
    // This is the second and last read of these lines: evict them first, so that L2 keeps
    // the score CTA's fresh loads, the partial outputs and the projection weights instead.
    const uint64_t pol_drop = l2_evict_first();
    BlockWindow win;
    int vt = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      for (int j = 0; j < tl.nb && ok; ++j) {
        const int blk = win.get(p, tl.b, tl.local0 + j, lane);
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
    // This warp arms each P slot for its next use (arrive + expected bytes) when it reaches
    // the block, so a slot's phase completes once the block and header have landed.
    int vt = 0, g = 0, t = 0;
    bool ok = true;
    while (ok && walk.next(tl)) {
      if (lane == 0)
        for (int j = 0; j < tl.nb; ++j) mbar_expect_tx(bar(kPFull + (g + j) % kPSlots), kSlotBytes);
      __syncwarp();
      // the header (in the first block's slot) has been read and any rescale applied
      ok = warp_wait(bar(kOReady), t & 1, ctl);
      if (!ok) {
        g += tl.nb;  // these slots were armed
        break;
      }
      for (int j = 0; j < tl.nb && ok; ++j, ++g) {
        const int slot = g % kPSlots;
        const int valid = min(kRows, tl.ntok - kRows * j);
        // each block's P . V starts as soon as that block has landed
        if (!warp_wait(bar(kPFull + slot), (g / kPSlots) & 1, ctl)) {
          ok = false;
          g += tl.nb - j;  // every slot of the tile was armed
          break;
        }
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
            const uint32_t pb = s_base + kV_P + slot * kSlotBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i)  // 16 rows per step; B MN-major: LBO = 64-dim slab
              mma_ss(tmem + 256 * dh, sdesc(pb + 32 * i, 16, 1024, 2),
                     sdesc(vb + 2048 * i, kSlabBytes, 1024, 2), kIdescPV,
                     (tl.first && j == 0 && i == 0) ? 0u : 1u);
            tc_commit(bar(kVEmpty + vs));
          }
          __syncwarp();
        }
        if (!ok) {
          g += tl.nb - j;  // every slot of the tile was armed
          break;
        }
        if (lane == 0) tc_commit(bar(kSlotDone + slot));
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar(kPvDone + (t & 1)));
      __syncwarp();
      ++t;
    }
    value_sent = g;  // P slot uses armed by this warp (for the teardown drain)
  } else if (!score && warp >= 2 && warp < 6) {
    // ------------------------------------------------ value: row sums, rescale, epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    int t = 0, g = 0;
    float l = 0.f;
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
      // the tile's first block carries the header: alpha (and the final maximum at the end)
      if (!warp_wait(bar(kPFull + g % kPSlots), (g / kPSlots) & 1, ctl)) break;
      const uint32_t hb = s_base + kV_P + (g % kPSlots) * kSlotBytes + kPBlockBytes;
      float alpha, m_last = 0.f;
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(alpha) : "r"(hb + 4u * h) : "memory");
      if (tl.last)
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(m_last) : "r"(hb + 4u * (kH + h)) : "memory");
      if (!tl.first && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_pv(t - 1)) break;  // (also keeps up with completions, see below)
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
      } else if (t >= 2 && !wait_pv(t - 2)) {
        // keep up with completions: OReady of tile t enables the P . V of tile t, whose
        // completion is the next phase of the barrier that tile t - 2 completed
        break;
      }
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOReady));
      // l: the sum of head h's bf16 P values, exactly what P . V consumes
      float rs0 = 0.f, rs1 = 0.f;
      for (int j = 0; j < tl.nb && ok; ++j) {
        if (j > 0) ok = warp_wait(bar(kPFull + (g + j) % kPSlots), ((g + j) / kPSlots) & 1, ctl);
        if (!ok) break;
        const uint32_t row = s_base + kV_P + ((g + j) % kPSlots) * kSlotBytes + (uint32_t)h * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t w0, w1, w2, w3;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                       : "r"(row + 16u * (uint32_t)u)
                       : "memory");
          rs0 += __uint_as_float(w0 << 16) + __uint_as_float(w0 & 0xffff0000u);
          rs1 += __uint_as_float(w1 << 16) + __uint_as_float(w1 & 0xffff0000u);
          rs0 += __uint_as_float(w2 << 16) + __uint_as_float(w2 & 0xffff0000u);
          rs1 += __uint_as_float(w3 << 16) + __uint_as_float(w3 & 0xffff0000u);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kSumDone + (g + j) % kPSlots));
      }
      if (!ok) break;
      l = (tl.first ? 0.f : l * alpha) + (rs0 + rs1);
      if (tl.last) {
        const float lse = (m_last + __log2f(l)) * 0.6931471805599453f;
        if (tl.slot < 0) {
          if (p.lse) p.lse[(size_t)tl.bt * kH + h] = lse;
        } else {
          p.part_lse[(size_t)tl.slot * kH + h] = lse;
        }
        if (!wait_pv(t)) break;
        tc_after();
        const float inv_l = 1.f / l;
        // O / l leaves through shared memory: each warp stages its 32 rows x 32 columns in a
        // 4 KB box (row = lane, 16-byte groups swizzled by row % 8), reads it back four rows
        // per instruction and stores whole 128-byte lines; the box is free again as soon as
        // the warp has read it, so no store is waited for. Kept in L2: the combine (partials)
        // and the output projection (O) read them next, after the rest of the cache has
        // streamed through.
        const uint64_t keep = l2_evict_last();
        float* dst = (tl.slot < 0 ? p.out + (size_t)tl.bt * kH * kR
                                  : p.part_o + (size_t)tl.slot * kH * kR) +
                     (size_t)(quad * 32 + (lane >> 3)) * kR + 4 * (lane & 7);
        const uint32_t box = s_base + kV_Out + (uint32_t)quad * kOutBoxBytes;
        const uint32_t wrow = box + (uint32_t)lane * 128;
        // read-back: instruction i takes rows 4i .. 4i + 3, lane: row 4i + lane / 8, 16-byte
        // group lane % 8, stored at group (lane % 8) ^ (row % 8) with row % 8 = lane / 8 for
        // even i and lane / 8 + 4 for odd i
        const uint32_t g = (uint32_t)((lane & 7) ^ (lane >> 3));
        const uint32_t rd_even = box + (uint32_t)(lane >> 3) * 128 + 16u * g;
        const uint32_t rd_odd = box + (uint32_t)(lane >> 3) * 128 + 16u * (g ^ 4u);
        // the next chunk's TMEM load is in flight while this chunk is staged and stored
        uint32_t o[32], nx[32];
        tmem_ld32(tq, o);
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
          if (ch + 1 < 16) tmem_ld32_async(tq + 32 * (ch + 1), nx);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                             wrow + 16u * (uint32_t)(u ^ (lane & 7))),
                         "f"(__uint_as_float(o[4 * u]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 1]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 2]) * inv_l),
                         "f"(__uint_as_float(o[4 * u + 3]) * inv_l)
                         : "memory");
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 x;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                         : "r"(((i & 1) ? rd_odd : rd_even) + 512u * (uint32_t)i)
                         : "memory");
            st_global_hint(dst + (size_t)(4 * i) * kR + 32 * ch, x, keep);
          }
          __syncwarp();  // the box is read before the next chunk overwrites it
          if (ch + 1 < 16) {
            tmem_wait_ld(nx);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = nx[i];
          }
        }
        tc_before();
      }
      g += tl.nb;
      ++t;
    }
  }

  // ---------------------------------------------------------------------- teardown
  // The score CTA tells the value CTA how many P blocks it sent, so that the value CTA can
  // wait (bounded) for any that are still landing in its shared memory before either exits.
  if (score && warp == 10 && lane == 0)
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_addr(saddr((void*)sent_count), peer)),
                 "r"(value_sent)
                 : "memory");
  tc_before();
  __syncthreads();
  tc_after();
  cluster_sync();  // the sent count is visible in the value CTA
  if (!score && warp == 1 && *abort_flag != 0) {
    // normal runs consumed every block; after an abort, wait for the blocks still in flight
    // (arming each slot use that the MMA warp did not reach)
    const int sent = *sent_count;
    for (int g = max(value_sent - kPSlots, 0); g < sent; ++g) {
      if (g >= value_sent) {
        if (lane == 0) mbar_expect_tx(bar(kPFull + g % kPSlots), kSlotBytes);
        __syncwarp();
      }
      drain_wait(bar(kPFull + g % kPSlots), (g / kPSlots) & 1, p.err);
    }
  }
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
  CUtensorMap kv, qm;
  if (!make_bf16_map(&kv, p.pool, kD, (uint64_t)p.num_blocks * kRows, kD * 2, kRows) ||
      !make_bf16_map(&qm, p.q, kD, (uint64_t)p.BT * kH, kD * 2, kH))
    return cudaErrorInvalidValue;
  // the shared-memory attribute applies to the device current when it is set: once per device
  static std::atomic<unsigned long long> attr_devices{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (!bit || !(attr_devices.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_devices.fetch_or(bit, std::memory_order_acq_rel);
  }
  return launch_pdl(attend_tc_kernel, dim3(2 * kRanges), dim3(kThreads), kSmemBytes, st, kv, qm,
                    p);
}

}  // namespace mla
