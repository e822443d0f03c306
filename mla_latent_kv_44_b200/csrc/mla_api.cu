// C ABI of libmla: argument validation, workspace carving and kernel dispatch.
// Every entry point validates synchronously before any CUDA call and only enqueues work.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"

using namespace mla;

namespace mla {
// decode_plan.cu: the merge behind mla_combine_partials
cudaError_t launch_combine_parts(const float* part_o, const float* part_lse, int parts, int n,
                                 int H, int r, float* out, float* lse, cudaStream_t st);
// front_tc.cu: the products behind mla_project
bool front_tc_supported(const mla_config& c, int K);
size_t front_part_bytes(const mla_config& c, int K, int n, const int* rows, int nseg,
                        bool norm);
cudaError_t launch_front_linear(const mla_config& c, const void* x, int n, int K, int ldx,
                                const void* const* w, const int* rows, void* const* out, int nseg,
                                int norm_seg, const float* gamma, float eps, void* part,
                                uint32_t* err, cudaStream_t st);
// fp8_cache.cu: the step's fp8 blocks expanded to bf16 for the tensor-core decode
cudaError_t launch_dequant_fp8(const uint8_t* pool, const float* row_scale, const int32_t* table,
                               const int32_t* seq_lens, int batch, int max_blocks, int num_blocks,
                               int bs, int D, void* out, int32_t* out_table, uint32_t* err,
                               cudaStream_t st);
// prefill_tc.cu: mla_prefill
bool prefill_tc_supported(const mla_config& c);
size_t prefill_workspace_bytes(const mla_config& c, int n);
cudaError_t launch_prefill(const mla_config& c, const void* q_nope, const void* q_rope,
                           const int32_t* pos, const void* rows, const void* w_uk,
                           const void* w_uv, const int32_t* cu, int batch, int max_seqlen, int n,
                           void* o, void* ws, uint32_t* err, cudaStream_t st);
}  // namespace mla

namespace {

bool valid_config(const mla_config* c) {
  if (!c) return false;
  if (c->num_heads < 1 || c->num_heads > 4096) return false;
  if (c->head_dim < 1 || c->head_dim > 1024) return false;
  if (c->head_dim_v < 1 || c->head_dim_v > 1024) return false;
  if (c->kv_rank < 32 || c->kv_rank > 1024 || c->kv_rank % 32 != 0) return false;
  if (c->rope_dim < 0 || c->rope_dim > 256 || c->rope_dim % 2 != 0) return false;
  if ((c->kv_rank + c->rope_dim) % 8 != 0) return false;
  if (c->block_size < 1) return false;
  if (c->dtype != MLA_F32 && c->dtype != MLA_BF16) return false;
  if (c->decode_kernel < MLA_DECODE_AUTO || c->decode_kernel > MLA_DECODE_TENSOR) return false;
  if (!std::isfinite(c->softmax_scale) || !(c->softmax_scale > 0.f)) return false;
  if (!std::isfinite(c->rope_base) || !(c->rope_base > 0.f)) return false;
  if (!std::isfinite(c->rms_eps) || c->rms_eps < 0.f) return false;
  return true;
}

mla_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

DecodeParams make_params(const mla_config* cfg, const void* q, const void* pool,
                         const int32_t* block_table, int32_t max_blocks, int32_t num_blocks,
                         const int32_t* seq_lens, int32_t batch, int32_t q_per_seq,
                         void* workspace, float* out_latent, float* lse, uint32_t* dev_err) {
  const int bt = batch * q_per_seq;
  const WorkspaceLayout L = workspace_layout(cfg->num_heads, cfg->kv_rank, bt);
  char* ws = static_cast<char*>(workspace);
  DecodeParams p;
  p.q = q;
  p.pool = pool;
  p.table = block_table;
  p.seq_lens = seq_lens;
  p.out = out_latent;
  p.lse = lse;
  p.err = dev_err;
  p.header = reinterpret_cast<int32_t*>(ws + L.header);
  p.range_begin = reinterpret_cast<int32_t*>(ws + L.range_begin);
  p.segments = reinterpret_cast<Segment*>(ws + L.segments);
  p.bt_slot0 = reinterpret_cast<int32_t*>(ws + L.bt_slot0);
  p.bt_nseg = reinterpret_cast<int32_t*>(ws + L.bt_nseg);
  p.bt_len = reinterpret_cast<int32_t*>(ws + L.bt_len);
  p.bt_chunk0 = reinterpret_cast<int32_t*>(ws + L.bt_chunk0);
  p.part_lse = reinterpret_cast<float*>(ws + L.part_lse);
  p.part_o = reinterpret_cast<float*>(ws + L.part_o);
  p.row_scale = nullptr;
  p.H = cfg->num_heads;
  p.r = cfg->kv_rank;
  p.dr = cfg->rope_dim;
  p.D = cfg->kv_rank + cfg->rope_dim;
  p.bs = cfg->block_size;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.batch = batch;
  p.T = q_per_seq;
  p.BT = bt;
  p.scale = cfg->softmax_scale;
  return p;
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
  }
  return "MLA_ERR_UNKNOWN";
}

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

}  // extern "C"

namespace {

// Byte offsets of mla_project's workspace: the K-split partial sums (shared by the two
// products, which run one after the other), then c_q' (n x q_rank, dtype).
struct FrontLayout {
  size_t part, cq, total;
};

bool front_valid(const mla_config* cfg, const mla_front_config* f, int32_t n) {
  return valid_config(cfg) && f && f->d_model >= 1 && f->d_model <= 57344 && f->q_rank >= 0 &&
         f->q_rank <= 12288 && std::isfinite(f->q_rms_eps) && f->q_rms_eps >= 0.f && n >= 0;
}

// Output rows of the products with x, in launch order: c_q (or q_nope), q_rope, c_kv, k_rope
// (the RoPE ones only when d_r > 0). Returns their count.
int front_rows(const mla_config& c, const mla_front_config& f, int* rows) {
  int nseg = 0;
  rows[nseg++] = f.q_rank > 0 ? f.q_rank : c.num_heads * c.head_dim;
  if (c.rope_dim > 0) rows[nseg++] = c.num_heads * c.rope_dim;
  rows[nseg++] = c.kv_rank;
  if (c.rope_dim > 0) rows[nseg++] = c.rope_dim;
  return nseg;
}

FrontLayout front_layout(const mla_config& c, const mla_front_config& f, int n) {
  int rows1[4];
  const int nseg = front_rows(c, f, rows1);
  size_t part = front_part_bytes(c, f.d_model, n, rows1, nseg, f.q_rank > 0);
  if (f.q_rank > 0) {
    const int rows3[1] = {c.num_heads * c.head_dim};
    part = std::max(part, front_part_bytes(c, f.q_rank, n, rows3, 1, false));
  }
  FrontLayout L;
  L.part = 0;
  L.cq = (part + 255) / 256 * 256;
  const size_t esz = c.dtype == MLA_BF16 ? 2 : 4;
  L.total = L.cq + ((size_t)n * f.q_rank * esz + 255) / 256 * 256;
  return L;
}

}  // namespace

extern "C" {

size_t mla_project_workspace_size(const mla_config* cfg, const mla_front_config* front,
                                  int32_t n_tokens) {
  if (!front_valid(cfg, front, n_tokens) || n_tokens == 0) return 0;
  return front_layout(*cfg, *front, n_tokens).total;
}

mla_status mla_project(const mla_config* cfg, const mla_front_config* front, const void* x,
                       const void* w_dq, const float* gamma_q, const void* w_uq,
                       const void* w_qr, const void* w_dkv, const void* w_kr, void* q_nope,
                       void* q_rope, void* ckv_raw, void* krope_raw, int32_t n_tokens,
                       void* workspace, size_t workspace_bytes, uint32_t* dev_err,
                       void* stream) {
  if (!front_valid(cfg, front, n_tokens)) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  const mla_config& c = *cfg;
  const mla_front_config& f = *front;
  const bool rope = c.rope_dim > 0, low = f.q_rank > 0;
  if (!x || !w_dq || !w_dkv || !q_nope || !ckv_raw || !workspace) return MLA_ERR_INVALID_ARG;
  if (low && (!w_uq || !gamma_q)) return MLA_ERR_INVALID_ARG;
  if (rope && (!w_qr || !w_kr || !q_rope || !krope_raw)) return MLA_ERR_INVALID_ARG;
  const FrontLayout L = front_layout(c, f, n_tokens);
  if (workspace_bytes < L.total || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  if (c.dtype == MLA_BF16) {
    if (!front_tc_supported(c, f.d_model) || (low && !front_tc_supported(c, f.q_rank)))
      return MLA_ERR_UNSUPPORTED;
    const void* ptrs[] = {x, w_dq, w_uq, w_qr, w_dkv, w_kr};
    for (const void* p : ptrs)
      if (p && !aligned(p, 16)) return MLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  const int H = c.num_heads, dh = c.head_dim;
  uint8_t* ws = (uint8_t*)workspace;
  void* cq = ws + L.cq;
  // the products with x: c_q (or q_nope), q_rope, c_kv, k_rope in one launch
  int rows1[4];
  const int nseg = front_rows(c, f, rows1);
  const void* w1[4] = {w_dq, rope ? w_qr : w_dkv, w_dkv, w_kr};
  void* out1[4] = {low ? cq : q_nope, rope ? q_rope : ckv_raw, ckv_raw, krope_raw};
  cudaError_t e = launch_front_linear(c, x, n_tokens, f.d_model, f.d_model, w1, rows1, out1, nseg,
                                      low ? 0 : -1, gamma_q, f.q_rms_eps, ws + L.part, dev_err,
                                      st);
  if (e == cudaSuccess && low) {
    const void* w3[1] = {w_uq};
    const int rows3[1] = {H * dh};
    void* out3[1] = {q_nope};
    e = launch_front_linear(c, cq, n_tokens, f.q_rank, f.q_rank, w3, rows3, out3, 1, -1,
                            nullptr, 0.f, ws + L.part, dev_err, st);
  }
  return from_cuda(e);
}

size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t n_tokens) {
  if (!valid_config(cfg) || n_tokens < 1) return 0;
  return prefill_workspace_bytes(*cfg, n_tokens);
}

mla_status mla_prefill(const mla_config* cfg, const void* q_nope, const void* q_rope,
                       const int32_t* pos, const void* rows, const void* w_uk, const void* w_uv,
                       const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                       int32_t n_tokens, void* o, void* workspace, size_t workspace_bytes,
                       uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || batch < 0 || n_tokens < 0 || max_seqlen < 0)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0 || n_tokens == 0) return MLA_OK;
  const mla_config& c = *cfg;
  const bool rope = c.rope_dim > 0;
  if (!q_nope || (rope && (!q_rope || !pos)) || !rows || !w_uk || !w_uv || !cu_seqlens || !o ||
      !workspace || max_seqlen < 1)
    return MLA_ERR_INVALID_ARG;
  // d_v: a warp's values on CUDA cores; d_h, d_r: the query is packed in 16-byte pieces
  const int vec = c.dtype == MLA_BF16 ? 8 : 4;
  if (c.head_dim_v > 256 || c.head_dim % vec != 0 || c.rope_dim % vec != 0)
    return MLA_ERR_UNSUPPORTED;
  if (!aligned(q_nope, 16) || (rope && !aligned(q_rope, 16))) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < prefill_workspace_bytes(c, n_tokens) || !aligned(workspace, 256))
    return MLA_ERR_WORKSPACE;
  if (c.dtype == MLA_BF16) {
    // the expansion of K and V streams the weights on the tensor cores (16-byte rows)
    if (c.kv_rank % 8 != 0 || (c.kv_rank + c.rope_dim) % 8 != 0) return MLA_ERR_UNSUPPORTED;
    const void* ptrs[] = {q_nope, q_rope, rows, w_uk, w_uv, o};
    for (const void* p : ptrs)
      if (p && !aligned(p, 16)) return MLA_ERR_INVALID_ARG;
  }
  return from_cuda(launch_prefill(c, q_nope, q_rope, pos, rows, w_uk, w_uv, cu_seqlens, batch,
                                  max_seqlen, n_tokens, o, workspace, dev_err,
                                  (cudaStream_t)stream));
}

mla_status mla_combine_partials(const mla_config* cfg, const float* part_latent,
                                const float* part_lse, int32_t parts, int32_t n,
                                float* out_latent, float* lse, void* stream) {
  if (!valid_config(cfg) || parts < 1 || parts > MLA_MAX_COMBINE_PARTS || n < 0)
    return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!part_latent || !part_lse || !out_latent) return MLA_ERR_INVALID_ARG;
  if (!aligned(part_latent, 16) || !aligned(out_latent, 16)) return MLA_ERR_INVALID_ARG;
  return from_cuda(launch_combine_parts(part_latent, part_lse, parts, n, cfg->num_heads,
                                        cfg->kv_rank, out_latent, lse, (cudaStream_t)stream));
}

mla_status mla_absorb_query(const mla_config* cfg, const void* q_nope, const void* q_rope,
                            const int32_t* pos, const void* w_uk, void* q_out, int32_t n_tokens,
                            uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || n_tokens < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!q_nope || !w_uk || !q_out || !pos || (cfg->rope_dim > 0 && !q_rope))
    return MLA_ERR_INVALID_ARG;
  if (n_tokens > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  const bool tc = cfg->decode_kernel != MLA_DECODE_SIMT && absorb_tc_supported(*cfg) &&
                  aligned(q_nope, 16) && aligned(w_uk, 16) && aligned(q_out, 16) &&
                  (cfg->rope_dim == 0 || aligned(q_rope, 16));
  if (cfg->decode_kernel == MLA_DECODE_TENSOR && !tc) return MLA_ERR_UNSUPPORTED;
  if (tc)
    return from_cuda(launch_absorb_tc(*cfg, q_nope, q_rope, pos, w_uk, q_out, n_tokens, dev_err,
                                      (cudaStream_t)stream));
  return from_cuda(launch_absorb(*cfg, q_nope, q_rope, pos, w_uk, q_out, n_tokens,
                                 (cudaStream_t)stream));
}

mla_status mla_append_latent(const mla_config* cfg, const void* ckv_raw, const void* krope_raw,
                             const float* gamma, const int32_t* seq_idx, const int32_t* pos,
                             const int32_t* block_table, int32_t batch, int32_t max_blocks,
                             void* pool, int32_t num_blocks, int32_t n_tokens, uint32_t* dev_err,
                             void* stream) {
  if (!valid_config(cfg) || n_tokens < 0 || batch < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!ckv_raw || (cfg->rope_dim > 0 && !krope_raw) || !gamma || !seq_idx || !pos ||
      !block_table || !pool || !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens > (1 << 26)) return MLA_ERR_UNSUPPORTED;
  return from_cuda(launch_append(*cfg, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table,
                                 batch, max_blocks, pool, num_blocks, n_tokens, dev_err,
                                 (cudaStream_t)stream));
}

size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t q_per_seq) {
  if (!valid_config(cfg) || batch < 1 || q_per_seq < 1) return 0;
  const int64_t bt = (int64_t)batch * q_per_seq;
  if (bt > (1 << 24)) return 0;
  return workspace_layout(cfg->num_heads, cfg->kv_rank, (int)bt).total;
}

mla_status mla_decode_stages(const mla_config* cfg, int32_t stages, const void* q,
                             const void* pool, const int32_t* block_table, int32_t max_blocks,
                             int32_t num_blocks, const int32_t* seq_lens, int32_t batch,
                             int32_t q_per_seq, void* workspace, size_t workspace_bytes,
                             float* out_latent, float* lse, uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || batch < 0 || q_per_seq < 1) return MLA_ERR_INVALID_ARG;
  if (stages & ~(MLA_STAGE_PLAN | MLA_STAGE_ATTEND | MLA_STAGE_COMBINE)) return MLA_ERR_INVALID_ARG;
  if (batch == 0 || stages == 0) return MLA_OK;
  if (!q || !pool || !block_table || !seq_lens || !workspace || !out_latent || !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  const int64_t bt = (int64_t)batch * q_per_seq;
  if (bt > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  const size_t need = mla_decode_workspace_size(cfg, batch, q_per_seq);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < need || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  if (!aligned(pool, 16) || !aligned(q, 16) || !aligned(out_latent, 16))
    return MLA_ERR_INVALID_ARG;

  bool use_tc;
  switch (cfg->decode_kernel) {
    case MLA_DECODE_SIMT: use_tc = false; break;
    case MLA_DECODE_TENSOR:
      if (!tc_supported(*cfg)) return MLA_ERR_UNSUPPORTED;
      use_tc = true;
      break;
    default: use_tc = tc_supported(*cfg); break;
  }

  const DecodeParams p = make_params(cfg, q, pool, block_table, max_blocks, num_blocks, seq_lens,
                                     batch, q_per_seq, workspace, out_latent, lse, dev_err);

  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (stages & MLA_STAGE_PLAN) e = launch_plan(p, st);
  if (e == cudaSuccess && (stages & MLA_STAGE_ATTEND))
    e = use_tc ? launch_attend_tc(*cfg, p, st) : launch_attend_simt(*cfg, p, st);
  if (e == cudaSuccess && (stages & MLA_STAGE_COMBINE)) e = launch_combine(p, st);
  return from_cuda(e);
}

mla_status mla_append_latent_fp8(const mla_config* cfg, const void* ckv_raw,
                                 const void* krope_raw, const float* gamma,
                                 const int32_t* seq_idx, const int32_t* pos,
                                 const int32_t* block_table, int32_t batch, int32_t max_blocks,
                                 uint8_t* pool, float* row_scale, int32_t num_blocks,
                                 int32_t n_tokens, uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || n_tokens < 0 || batch < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!ckv_raw || (cfg->rope_dim > 0 && !krope_raw) || !gamma || !seq_idx || !pos ||
      !block_table || !pool || !row_scale || !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens > (1 << 26)) return MLA_ERR_UNSUPPORTED;
  return from_cuda(launch_append_fp8(*cfg, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table,
                                     batch, max_blocks, pool, row_scale, num_blocks, n_tokens,
                                     dev_err, (cudaStream_t)stream));
}

// The fp8 decode's workspace: mla_decode's, then (tensor-core path) the scratch block table
// (batch x max_blocks int32) and the scratch bf16 pool (batch x max_blocks blocks).
struct Fp8Layout {
  size_t table, pool, total;
  bool tc;
};

Fp8Layout fp8_layout(const mla_config& c, int batch, int q_per_seq, int max_blocks) {
  Fp8Layout L{};
  const size_t dec = mla_decode_workspace_size(&c, batch, q_per_seq);
  L.tc = c.decode_kernel != MLA_DECODE_SIMT && tc_supported(c);
  L.table = (dec + 255) / 256 * 256;
  L.pool = L.table + ((size_t)batch * max_blocks * 4 + 255) / 256 * 256;
  L.total = L.tc ? L.pool + (size_t)batch * max_blocks * c.block_size *
                                (c.kv_rank + c.rope_dim) * 2
                 : dec;
  return L;
}

size_t mla_decode_fp8_workspace_size(const mla_config* cfg, int32_t batch, int32_t q_per_seq,
                                     int32_t max_blocks) {
  if (mla_decode_workspace_size(cfg, batch, q_per_seq) == 0 || max_blocks < 1) return 0;
  return fp8_layout(*cfg, batch, q_per_seq, max_blocks).total;
}

mla_status mla_decode_fp8(const mla_config* cfg, const void* q, const uint8_t* pool,
                          const float* row_scale, const int32_t* block_table, int32_t max_blocks,
                          int32_t num_blocks, const int32_t* seq_lens, int32_t batch,
                          int32_t q_per_seq, void* workspace, size_t workspace_bytes,
                          float* out_latent, float* lse, uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || batch < 0 || q_per_seq < 1) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q || !pool || !row_scale || !block_table || !seq_lens || !workspace || !out_latent ||
      !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  const int64_t bt = (int64_t)batch * q_per_seq;
  if (bt > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  if (mla_decode_workspace_size(cfg, batch, q_per_seq) == 0) return MLA_ERR_INVALID_ARG;
  const Fp8Layout L = fp8_layout(*cfg, batch, q_per_seq, max_blocks);
  if (workspace_bytes < L.total || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  if (!aligned(pool, 16) || !aligned(q, 16) || !aligned(out_latent, 16))
    return MLA_ERR_INVALID_ARG;
  if ((int64_t)batch * max_blocks > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (L.tc) {
    // the step's blocks in bf16, then the tensor-core decode over them
    uint8_t* ws = (uint8_t*)workspace;
    int32_t* table_s = (int32_t*)(ws + L.table);
    void* pool_s = ws + L.pool;
    e = launch_dequant_fp8(pool, row_scale, block_table, seq_lens, batch, max_blocks, num_blocks,
                           cfg->block_size, cfg->kv_rank + cfg->rope_dim, pool_s, table_s,
                           dev_err, st);
    const DecodeParams p = make_params(cfg, q, pool_s, table_s, max_blocks, batch * max_blocks,
                                       seq_lens, batch, q_per_seq, workspace, out_latent, lse,
                                       dev_err);
    if (e == cudaSuccess) e = launch_plan(p, st);
    if (e == cudaSuccess) e = launch_attend_tc(*cfg, p, st);
    if (e == cudaSuccess) e = launch_combine(p, st);
    return from_cuda(e);
  }
  DecodeParams p = make_params(cfg, q, pool, block_table, max_blocks, num_blocks, seq_lens, batch,
                               q_per_seq, workspace, out_latent, lse, dev_err);
  p.row_scale = row_scale;
  e = launch_plan(p, st);
  if (e == cudaSuccess) e = launch_attend_simt_fp8(*cfg, p, st);
  if (e == cudaSuccess) e = launch_combine(p, st);
  return from_cuda(e);
}

mla_status mla_decode(const mla_config* cfg, const void* q, const void* pool,
                      const int32_t* block_table, int32_t max_blocks, int32_t num_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t q_per_seq, void* workspace,
                      size_t workspace_bytes, float* out_latent, float* lse, uint32_t* dev_err,
                      void* stream) {
  return mla_decode_stages(cfg, MLA_STAGE_PLAN | MLA_STAGE_ATTEND | MLA_STAGE_COMBINE, q, pool,
                           block_table, max_blocks, num_blocks, seq_lens, batch, q_per_seq,
                           workspace, workspace_bytes, out_latent, lse, dev_err, stream);
}

mla_status mla_output(const mla_config* cfg, const float* out_latent, const void* w_uv, void* o,
                      int32_t n_tokens, uint32_t* dev_err, void* stream) {
  if (!valid_config(cfg) || n_tokens < 0) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!out_latent || !w_uv || !o) return MLA_ERR_INVALID_ARG;
  if (n_tokens > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  const bool tc = cfg->decode_kernel != MLA_DECODE_SIMT && output_tc_supported(*cfg) &&
                  aligned(out_latent, 16) && aligned(w_uv, 16);
  if (cfg->decode_kernel == MLA_DECODE_TENSOR && !tc) return MLA_ERR_UNSUPPORTED;
  if (tc)
    return from_cuda(launch_output_tc(*cfg, out_latent, w_uv, o, n_tokens, dev_err,
                                      (cudaStream_t)stream));
  return from_cuda(launch_output(*cfg, out_latent, w_uv, o, n_tokens, (cudaStream_t)stream));
}

mla_status mla_decode_step(const mla_config* cfg, const void* q_nope, const void* q_rope,
                           const void* w_uk, const void* ckv_raw, const void* krope_raw,
                           const float* gamma, const int32_t* seq_idx, const int32_t* pos,
                           const int32_t* block_table, int32_t max_blocks, void* pool,
                           int32_t num_blocks, const int32_t* seq_lens, int32_t batch,
                           int32_t q_per_seq, void* q_work, void* workspace,
                           size_t workspace_bytes, float* out_latent, float* lse,
                           const void* w_uv, void* o, uint32_t* dev_err, void* stream) {
  // Every argument is checked as the four calls check theirs, before anything is launched.
  if (!valid_config(cfg) || batch < 0 || q_per_seq < 1) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const bool rope = cfg->rope_dim > 0;
  if (!q_nope || (rope && !q_rope) || !w_uk || !ckv_raw || (rope && !krope_raw) || !gamma ||
      !seq_idx || !pos || !block_table || !pool || !seq_lens || !q_work || !workspace ||
      !out_latent || !w_uv || !o || !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  const int64_t n64 = (int64_t)batch * q_per_seq;
  if (n64 > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  const int n = (int)n64;
  const size_t need = mla_decode_workspace_size(cfg, batch, q_per_seq);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < need || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  if (!aligned(pool, 16) || !aligned(q_work, 16) || !aligned(out_latent, 16))
    return MLA_ERR_INVALID_ARG;
  const bool simt = cfg->decode_kernel == MLA_DECODE_SIMT;
  const bool attend_tc = !simt && tc_supported(*cfg);
  if (cfg->decode_kernel == MLA_DECODE_TENSOR && !tc_supported(*cfg)) return MLA_ERR_UNSUPPORTED;
  // the fused launches: tensor-core absorb, attention and output, 16-byte aligned operands
  const bool fused = attend_tc && absorb_tc_supported(*cfg) && output_tc_supported(*cfg) &&
                     aligned(q_nope, 16) && aligned(w_uk, 16) && aligned(q_rope, 16) &&
                     aligned(w_uv, 16);
  cudaStream_t st = (cudaStream_t)stream;
  if (!fused) {
    // the four calls' own kernels, in order (each validates as above and cannot fail here)
    mla_status s = mla_absorb_query(cfg, q_nope, q_rope, pos, w_uk, q_work, n, dev_err, stream);
    if (s == MLA_OK)
      s = mla_append_latent(cfg, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table, batch,
                            max_blocks, pool, num_blocks, n, dev_err, stream);
    if (s == MLA_OK)
      s = mla_decode(cfg, q_work, pool, block_table, max_blocks, num_blocks, seq_lens, batch,
                     q_per_seq, workspace, workspace_bytes, out_latent, lse, dev_err, stream);
    if (s == MLA_OK) s = mla_output(cfg, out_latent, w_uv, o, n, dev_err, stream);
    return s;
  }
  const DecodeParams p = make_params(cfg, q_work, pool, block_table, max_blocks, num_blocks,
                                     seq_lens, batch, q_per_seq, workspace, out_latent, lse,
                                     dev_err);
  cudaError_t e = launch_step_prep(*cfg, q_nope, q_rope, pos, w_uk, q_work, n, ckv_raw,
                                   krope_raw, gamma, seq_idx, p, pool, st);
  if (e == cudaSuccess) e = launch_attend_tc(*cfg, p, st);
  if (e == cudaSuccess) e = launch_combine(p, st);
  if (e == cudaSuccess) e = launch_output_tc(*cfg, out_latent, w_uv, o, n, dev_err, st);
  return from_cuda(e);
}

}  // extern "C"
