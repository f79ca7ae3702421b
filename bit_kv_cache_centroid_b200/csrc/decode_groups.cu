// decode_groups.cu — instantiations of the split decode kernel for caches
// whose (scale, zero) groups span 64 or 128 channels (decode_split.cuh); the
// 32-channel kernels are instantiated in decode.cu. A separate file so that
// the two sets compile in parallel.
#include "decode_split.cuh"

namespace kv2 {
namespace dsplit {

#define KV2_DSPLIT_INSTANTIATE(D, U16, GS)                                                  \
  template cudaError_t launch_g<D, U16, GS>(int, const SplitParams&, int, cudaStream_t); \
  template int ctas_per_sm_g<D, U16, GS>(int, int, int);
KV2_DSPLIT_GROUP_INSTANCES(KV2_DSPLIT_INSTANTIATE)

}  // namespace dsplit
}  // namespace kv2
