// Local attention backward on the tensor cores (bf16): see the kernels below.
#include "sm100.cuh"

namespace uly {

uly_status attn_bf16_bwd_launch(const uly_attn_desc *, const HeadGeom &, const MaskInfo &,
                                const void *, const void *, const void *, const void *,
                                const float *, const void *, void *, void *, void *, float *,
                                cudaStream_t) {
  return ULY_ERR_UNSUPPORTED;
}

}  // namespace uly
