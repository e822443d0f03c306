// tcgen05 tensor-core attention stage of mla_decode (bf16, H=128, r=512, d_r=64, 64-row blocks).
#include "common.cuh"

namespace mla {

bool tc_supported(const mla_config& c) {
  (void)c;
  return false;
}

cudaError_t launch_attend_tc(const mla_config& c, const DecodeParams& p, cudaStream_t st) {
  (void)c;
  (void)p;
  (void)st;
  return cudaErrorNotSupported;
}

}  // namespace mla
