// tcgen05 tensor-core attention stage of mla_decode (bf16 cache, H = 128, r = 512, d_r = 64,
// 64-row cache blocks), for sm_100a.
//
// Absorbed decode ("DeepSeek MLA, Built From the Paper", 3 Matrix absorption; "Build a DeepSeek
// Model from Scratch" ch. 3, score = content score + position score; "MLA from scratch in
// PyTorch", Absorbing projections: attend directly to latents). For one query token the 128
// heads are the M = 128 rows of two dense contractions against the shared cache tile:
//   S = Q . K^T      (M = 128 heads, N = 64 rows, K = 576 = [c_kv || k_rope])
//   O += P . V       (M = 128 heads, N = 512 latent dims, K = 64 rows; V = the c_kv part of K)
// so each cache tile is read from HBM once and serves both products.
//
// O for 128 heads x 512 dims in fp32 is 256 KB: all of one SM's tensor memory. A cluster of two
// CTAs therefore shares every work range. CTA c loads only its half of each row -- latent dims
// [256c, 256c + 256) and RoPE dims [32c, 32c + 32) -- so the pair reads each cache byte once:
//   * both CTAs compute a partial S over their 288 dims (Q half resident in TMEM as the A
//     operand), swap the fp32 partials through distributed shared memory (st.async into the
//     peer's double-buffered inbox, completing on the peer's own mbarrier) and add them; IEEE
//     addition commutes, so both hold bit-identical S and take identical softmax decisions;
//   * each CTA accumulates P . V for its own 256 latent dims in TMEM (256 columns).
// TMEM columns: O [0,256), S [256,320), P [320,352) (bf16 pairs), Q [352,496) (bf16 pairs).
//
// Warp roles: warp 0 issues TMA loads into a 4-stage ring, warp 1 issues the MMAs (QK of tile
// t+1 before PV of tile t, so the tensor pipe works while the softmax warps work), warps 2-5
// (one TMEM lane per head) run the online softmax in exp2 units with a lazy rescale of O (only
// when the running max grows by more than 2^8), and the epilogue. Every wait is bounded: on
// timeout the kernel sets MLA_DEV_WAIT_TIMEOUT, drains its own copies and MMAs, frees TMEM and
// returns. No TMA multicast is used.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace mla {
namespace {

constexpr int kH = 128;
constexpr int kR = 512;
constexpr int kDR = 64;
constexpr int kD = kR + kDR;
constexpr int kRows = 64;                                 // rows per tile = block = chunk
constexpr int kStages = 4;
constexpr int kSlabBytes = kRows * 64 * 2;                // 64 rows x 64 dims bf16: 8 KB
constexpr int kRopeBytes = kRows * 32 * 2;                // 64 rows x 32 dims bf16: 4 KB
constexpr int kStageBytes = 4 * kSlabBytes + kRopeBytes;  // 36 KB
constexpr int kInboxBytes = kH * kRows * 4;               // 128 x 64 fp32: 32 KB per slot
constexpr int kInboxSlots = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352;
constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait

enum Bar {
  kFull = 0,
  kEmpty = kFull + kStages,
  kSFull = kEmpty + kStages,
  kSFree, kPFull, kPvDone, kQFull, kOFree, kXFull, kFinal = kXFull + kInboxSlots, kNumBars
};
constexpr int kBarOff = kStages * kStageBytes + kInboxSlots * kInboxBytes;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // +1024: manual alignment

// instruction descriptors, kind::f16: bf16 A and B, fp32 D, A K-major
constexpr uint32_t idesc(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc(128, 64, 0);
constexpr uint32_t kIdescPV = idesc(128, 256, 1);

// ------------------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// 16 bytes into the peer CTA's shared memory; completes bytes on the peer's mbarrier.
__device__ __forceinline__ void st_async_peer(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d, uint32_t peer_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d), "r"(peer_bar)
      : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                         int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst), "l"(map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[tmem] . B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t id,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d), "r"(a), "l"(bdesc),
      "r"(id), "r"(acc)
      : "memory");
}
// 32 consecutive columns of this thread's TMEM lane, waited before returning.
__device__ __forceinline__ void tmem_ld32(uint32_t ta, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(ta)
      : "memory");
}
// 64 consecutive columns, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t ta, uint32_t (&v)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,"
      "%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]), "=r"(v[32]), "=r"(v[33]), "=r"(v[34]),
        "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]), "=r"(v[40]), "=r"(v[41]),
        "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]), "=r"(v[48]),
        "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]),
        "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]),
        "=r"(v[63])
      : "r"(ta), "r"(ta + 32u)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t ta, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(ta),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t ta, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(ta),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor (Blackwell version 1): start, leading and stride byte
// offsets in 16-byte units, swizzle mode in bits 61-63 (2 = 128-byte, 4 = 64-byte).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                          uint32_t swz) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | ((uint64_t)swz << 61);
}

struct Ctl {
  uint32_t* err;
  volatile int* abort;
};

// Warp-collective bounded wait; the result is the same in all 32 lanes.
__device__ __noinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Ctl& c) {
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

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_ckv,
                 const __grid_constant__ CUtensorMap tm_rope, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s_base = saddr(smem);
  const uint32_t s_inbox = s_base + kStages * kStageBytes;
  const uint32_t s_bar = s_base + kBarOff;
  uint32_t* tmem_slot = (uint32_t*)(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = (volatile int*)(smem + kBarOff + kNumBars * 8 + 4);
  auto bar = [&](int i) { return s_bar + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const Ctl ctl{p.err, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(kFull + i), 1);
      mbar_init(bar(kEmpty + i), 1);
    }
    mbar_init(bar(kSFull), 1);
    mbar_init(bar(kSFree), 4);
    mbar_init(bar(kPFull), 4);
    mbar_init(bar(kPvDone), 1);
    mbar_init(bar(kQFull), 4);
    mbar_init(bar(kOFree), 4);
    for (int i = 0; i < kInboxSlots; ++i) mbar_init(bar(kXFull + i), 1);
    mbar_init(bar(kFinal), 1);
    // each inbox slot expects one partial score tile (from the peer) per phase
    for (int i = 0; i < kInboxSlots; ++i) mbar_expect_tx(bar(kXFull + i), kInboxBytes);
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
  cluster_sync();  // barriers of both CTAs initialised before any remote store
  const uint32_t tmem = *tmem_slot;

  // this pair's segments
  const int q = blockIdx.x >> 1;
  int sb = 0, se = 0;
  if (q < p.header[1]) {
    sb = p.range_begin[q];
    se = p.range_begin[q + 1];
  }

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    int t = 0;
    bool ok = true;
    for (int s = sb; ok && s < se; ++s) {
      const Segment sg = p.segments[s];
      const int b = sg.bt / p.T;
      const int n = sg.chunk_hi - sg.chunk_lo;
      const int32_t* trow =
          p.table + (size_t)b * p.max_blocks + (sg.chunk_lo - p.bt_chunk0[sg.bt]);
      for (int base = 0; ok && base < n; base += 32) {
        // block ids of the next 32 chunks, one per lane
        int my = 0;
        if (base + lane < n) {
          my = trow[base + lane];
          if (my < 0 || my >= p.num_blocks) {
            set_error(p.err, MLA_DEV_OOB_BLOCK);
            my = 0;
          }
        }
        const int cnt = min(32, n - base);
        for (int i = 0; i < cnt; ++i) {
          const int blk = __shfl_sync(0xffffffffu, my, i);
          const int stage = t % kStages;
          if (t >= kStages && !warp_wait(bar(kEmpty + stage), ((t / kStages) - 1) & 1, ctl)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            const uint32_t dst = s_base + stage * kStageBytes;
            const uint32_t fb = bar(kFull + stage);
            mbar_expect_tx(fb, kStageBytes);
            for (int k = 0; k < 4; ++k)
              tma_load(dst + k * kSlabBytes, &tm_ckv, fb, 256 * (int)rank + 64 * k, blk * kRows);
            tma_load(dst + 4 * kSlabBytes, &tm_rope, fb, kR + 32 * (int)rank, blk * kRows);
          }
          __syncwarp();
          ++t;
        }
      }
    }
    // drain: every issued load has landed before the CTA may exit
    for (int k = 1; k <= kStages && k <= t; ++k) {
      const int tt = t - k;
      const uint64_t t0 = globaltimer();
      bool done = false;
      while (!done && globaltimer() - t0 < kTimeoutNs)
        done = __all_sync(0xffffffffu, mbar_try(bar(kFull + tt % kStages), (tt / kStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    int t = 0, seg_i = 0;
    int prev_stage = 0, prev_seg = 0;
    bool prev_first = false, have_prev = false, ok = true;
    auto issue_pv = [&](int tp) -> bool {
      if (!warp_wait(bar(kPFull), tp & 1, ctl)) return false;
      if (prev_first && prev_seg > 0 && !warp_wait(bar(kOFree), (prev_seg - 1) & 1, ctl))
        return false;
      tc_after();
      if (lane == 0) {
        const uint32_t vbase = s_base + prev_stage * kStageBytes;
#pragma unroll
        for (int k = 0; k < 4; ++k)  // 16 rows per step; MN-major B: LBO = 64-dim slab, SBO = 8 rows
          mma_ts(tmem + kColO, tmem + kColP + 8 * k, sdesc(vbase + k * 2048, kSlabBytes, 1024, 2),
                 kIdescPV, (prev_first && k == 0) ? 0u : 1u);
        tc_commit(bar(kPvDone));
        tc_commit(bar(kEmpty + prev_stage));
      }
      __syncwarp();
      return true;
    };
    for (int s = sb; ok && s < se; ++s, ++seg_i) {
      const Segment sg = p.segments[s];
      const int chunk0 = p.bt_chunk0[sg.bt];
      const int len = p.bt_len[sg.bt];
      for (int c = sg.chunk_lo; c < sg.chunk_hi; ++c) {
        const bool first = (c == sg.chunk_lo);
        const int valid = min(kRows, len - (c - chunk0) * kRows);
        const int stage = t % kStages;
        ok = warp_wait(bar(kFull + stage), (t / kStages) & 1, ctl);
        if (ok && first) ok = warp_wait(bar(kQFull), seg_i & 1, ctl);
        if (ok && t > 0) ok = warp_wait(bar(kSFree), (t - 1) & 1, ctl);
        if (!ok) break;
        const uint32_t kbase = s_base + stage * kStageBytes;
        if (valid < kRows) {
          // rows past the sequence end: zero their latent part so 0 * garbage never enters P . V
          uint8_t* st = smem + stage * kStageBytes;
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
#pragma unroll
          for (int k = 0; k < 16; ++k)  // latent half: four 64-dim slabs, 16 dims per step
            mma_ts(tmem + kColS, tmem + kColQ + 8 * k,
                   sdesc(kbase + (k >> 2) * kSlabBytes + (k & 3) * 32, 16, 1024, 2), kIdescQK,
                   k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < 2; ++k)  // RoPE half: 32 dims, 64-byte swizzle
            mma_ts(tmem + kColS, tmem + kColQ + 128 + 8 * k,
                   sdesc(kbase + 4 * kSlabBytes + k * 32, 16, 512, 4), kIdescQK, 1u);
          tc_commit(bar(kSFull));
        }
        __syncwarp();
        if (have_prev && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
        prev_stage = stage;
        prev_first = first;
        prev_seg = seg_i;
        have_prev = true;
        ++t;
      }
    }
    if (ok && have_prev) issue_pv(t - 1);
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;  // scores in log2 units
    const __nv_bfloat16* Q = (const __nv_bfloat16*)p.q;
    const uint32_t row_off = (uint32_t)h * (kRows * 4);
    const uint32_t peer_inbox = peer_addr(s_inbox, peer);
    uint32_t peer_xfull[kInboxSlots];
#pragma unroll
    for (int i = 0; i < kInboxSlots; ++i) peer_xfull[i] = peer_addr(bar(kXFull + i), peer);
    const int swz = h & 15;

    auto load_q = [&](int bt) {
      const uint4* src = (const uint4*)(Q + ((size_t)bt * kH + h) * kD);
      uint32_t w[32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = src[(256 * rank + 64 * ch) / 8 + i];
          w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
        tmem_st32(tl + kColQ + 32 * ch, w);
      }
      uint32_t wr[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = src[(kR + 32 * rank) / 8 + i];
        wr[4 * i] = v.x; wr[4 * i + 1] = v.y; wr[4 * i + 2] = v.z; wr[4 * i + 3] = v.w;
      }
      tmem_st16(tl + kColQ + 128, wr);
      tmem_wait_st();
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kQFull));
    };

    int t = 0;
    float m_ref = 0.f, l = 0.f;
    bool ok = true;
    if (sb < se) load_q(p.segments[sb].bt);
    for (int s = sb; ok && s < se; ++s) {
      const Segment sg = p.segments[s];
      const int chunk0 = p.bt_chunk0[sg.bt];
      const int len = p.bt_len[sg.bt];
      for (int c = sg.chunk_lo; ok && c < sg.chunk_hi; ++c) {
        const bool first = (c == sg.chunk_lo), last = (c == sg.chunk_hi - 1);
        const int valid = min(kRows, len - (c - chunk0) * kRows);

        // own partial scores
        if (!warp_wait(bar(kSFull), t & 1, ctl)) { ok = false; break; }
        tc_after();
        uint32_t sv[64];
        tmem_ld64(tl + kColS, sv);
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kSFree));

        // swap partials with the other CTA: write into its inbox slot, read ours
        const int slot = t & 1;
        const uint32_t pdst = peer_inbox + (uint32_t)slot * kInboxBytes + row_off;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          st_async_peer(pdst + 16u * (uint32_t)(u ^ swz), sv[4 * u], sv[4 * u + 1], sv[4 * u + 2],
                        sv[4 * u + 3], peer_xfull[slot]);
        if (!warp_wait(bar(kXFull + slot), (t >> 1) & 1, ctl)) { ok = false; break; }
        float x[64];
        const uint32_t mine = s_inbox + (uint32_t)slot * kInboxBytes + row_off;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(mine + 16u * (uint32_t)(u ^ swz))
                       : "memory");
          x[4 * u] = __uint_as_float(sv[4 * u]) + __uint_as_float(v.x);
          x[4 * u + 1] = __uint_as_float(sv[4 * u + 1]) + __uint_as_float(v.y);
          x[4 * u + 2] = __uint_as_float(sv[4 * u + 2]) + __uint_as_float(v.z);
          x[4 * u + 3] = __uint_as_float(sv[4 * u + 3]) + __uint_as_float(v.w);
        }
        // this slot's next use is tile t + 2; the peer can only write it after receiving our
        // partial of tile t + 1, so re-arming now cannot race with this tile's reads
        if (threadIdx.x == 64) mbar_expect_tx(bar(kXFull + slot), kInboxBytes);

        // online softmax in log2 units, lazy rescale of O
        float mt = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          x[k] = (k < valid) ? x[k] * c2 : -INFINITY;
          mt = fmaxf(mt, x[k]);
        }
        float alpha = 1.f;
        bool rescale = false;
        if (first) {
          m_ref = mt;
          l = 0.f;
        } else if (mt > m_ref + 8.f) {
          alpha = ex2(m_ref - mt);
          m_ref = mt;
          rescale = true;
        }
        float rs = 0.f;
        uint32_t pw[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2(x[2 * k] - m_ref);
          const float p1 = ex2(x[2 * k + 1] - m_ref);
          rs += p0;
          rs += p1;
          pw[k] = pack_bf16(p0, p1);
        }
        l = l * alpha + rs;

        // P . V of the previous tile must be done before P and O are touched
        if (t > 0 && !warp_wait(bar(kPvDone), (t - 1) & 1, ctl)) { ok = false; break; }
        tc_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t o[32];
            tmem_ld32(tl + kColO + 32 * ch, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + kColO + 32 * ch, o);
          }
        }
        tmem_st32(tl + kColP, pw);
        tmem_wait_st();
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kPFull));
        ++t;

        if (last) {
          // next segment's query goes in while this segment drains
          if (s + 1 < se) load_q(p.segments[s + 1].bt);
          if (!warp_wait(bar(kPvDone), (t - 1) & 1, ctl)) { ok = false; break; }
          tc_after();
          const float inv_l = 1.f / l;
          const float lse = (m_ref + __log2f(l)) * 0.6931471805599453f;
          float* dst = (sg.slot < 0 ? p.out + ((size_t)sg.bt * kH + h) * kR
                                    : p.part_o + ((size_t)sg.slot * kH + h) * kR) +
                       256 * rank;
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t o[32];
            tmem_ld32(tl + kColO + 32 * ch, o);
            float4* d4 = (float4*)(dst + 32 * ch);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l,
                                  __uint_as_float(o[4 * i + 1]) * inv_l,
                                  __uint_as_float(o[4 * i + 2]) * inv_l,
                                  __uint_as_float(o[4 * i + 3]) * inv_l);
          }
          if (rank == 0) {
            if (sg.slot < 0) {
              if (p.lse) p.lse[(size_t)sg.bt * kH + h] = lse;
            } else {
              p.part_lse[(size_t)sg.slot * kH + h] = lse;
            }
          }
          tc_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kOFree));
        }
      }
    }
  }

  // ---------------------------------------------------------------------- teardown
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 1) {
    if (lane == 0) tc_commit(bar(kFinal));  // completes once every MMA issued here is done
    __syncwarp();
    const uint64_t t0 = globaltimer();
    bool done = false;
    while (!done && globaltimer() - t0 < kTimeoutNs)
      done = __all_sync(0xffffffffu, mbar_try(bar(kFinal), 0));
    if (!done && lane == 0) set_error(p.err, MLA_DEV_WAIT_TIMEOUT);
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
  cluster_sync();  // the peer no longer touches this CTA's shared memory
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* pool, int num_blocks, uint32_t box_cols,
              CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)num_blocks * kRows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {box_cols, (cuuint32_t)kRows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.num_heads == kH && c.kv_rank == kR && c.rope_dim == kDR &&
         c.block_size == kRows;
}

cudaError_t launch_attend_tc(const mla_config& c, const DecodeParams& p, cudaStream_t st) {
  (void)c;
  CUtensorMap ckv, rope;
  if (!make_map(&ckv, p.pool, p.num_blocks, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&rope, p.pool, p.num_blocks, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  attend_tc_kernel<<<2 * kRanges, kThreads, kSmemBytes, st>>>(ckv, rope, p);
  return cudaGetLastError();
}

}  // namespace mla
