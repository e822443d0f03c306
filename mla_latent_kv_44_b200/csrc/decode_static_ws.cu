// mla_decode_static_workspace: mla_decode with its workspace in a fixed device array owned by
// the library, for callers that cannot allocate device memory themselves.
//
// Who needs it: a caller that has no device allocator of its own (a plain C or embedded host
// program that links only this library and the CUDA runtime), or one that must not call
// cudaMalloc in the middle of a decode loop because cudaMalloc synchronises the device and
// would stall every other stream. Such a caller still passes the inputs and outputs; the
// schedule and the partial results live in g_decode_scratch below.
//
// The array is MLA_STATIC_WORKSPACE_BYTES (40 MiB) of device memory on every GPU that loads
// this library, held until the process exits. Its contents persist from call to call, and
// nothing in it has to start at zero: each call's planner rewrites the whole schedule before
// the attention and combine kernels read it, and partial results are written before they are
// read. Calls that overlap on the GPU (other streams, other host threads) share the array and
// race; serialise them.
#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[MLA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the symbol's name
// is only a host-side stand-in, so the address is fetched once per device, with that device
// current, and reused; the first call on a device does this set-up.
mla_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_static_workspace(const mla_config* cfg, const void* q,
                                                  const void* pool, const int32_t* block_table,
                                                  int32_t max_blocks, int32_t num_blocks,
                                                  const int32_t* seq_lens, int32_t batch,
                                                  int32_t q_per_seq, float* out_latent,
                                                  float* lse, uint32_t* dev_err, void* stream) {
  // The checks of mla_decode, in its order, so that both entry points return the same status
  // for the same arguments (a configuration is valid iff it has a workspace size at batch 1);
  // then the one check of this entry point: the workspace must fit the array.
  if (mla_decode_workspace_size(cfg, 1, 1) == 0 || batch < 0 || q_per_seq < 1)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q || !pool || !block_table || !seq_lens || !out_latent || !dev_err)
    return MLA_ERR_INVALID_ARG;
  if (max_blocks < 1 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if ((int64_t)batch * q_per_seq > (1 << 24)) return MLA_ERR_UNSUPPORTED;
  const size_t need = mla_decode_workspace_size(cfg, batch, q_per_seq);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > (size_t)MLA_STATIC_WORKSPACE_BYTES) return MLA_ERR_WORKSPACE;
  void* ws = nullptr;
  const mla_status st = scratch_address(&ws);
  if (st != MLA_OK) return st;
  return mla_decode(cfg, q, pool, block_table, max_blocks, num_blocks, seq_lens, batch,
                    q_per_seq, ws, (size_t)MLA_STATIC_WORKSPACE_BYTES, out_latent, lse, dev_err,
                    stream);
}
