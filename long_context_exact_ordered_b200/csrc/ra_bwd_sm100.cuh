// sm_100a backward (bf16): placeholder until the tensor-core kernel lands.
#pragma once

#include "ra_common.cuh"
#include "ra_simt.cuh"

namespace ra {

template <int D>
int launch_bwd_sm100(const ra_tensor*, const ra_tensor*, const ra_tensor*, const ra_tensor*, const ra_tensor*,
                     const MaskArgs&, const RingDesc&, const int4*, float*, float*, ra_tensor*, ra_tensor*,
                     ra_tensor*, cudaStream_t) {
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
