// Tensor-core path (M > 32): placeholder until the tcgen05 kernels land.
#include "common.cuh"
#include "kernels.h"

namespace mxg {

bool plan_w4a16_tc(int, int, int, int, int, TcPlan *) { return false; }
cudaError_t launch_w4a16_tc(const TcPlan &, const void *, const void *, int, int, int, int, void *,
                            void *, cudaStream_t)
{
    return cudaErrorNotSupported;
}
bool plan_mxfp8_tc(int, int, int, int, TcPlan *) { return false; }
cudaError_t launch_mxfp8_tc(const TcPlan &, const void *, const uint8_t *, const uint8_t *, int, int,
                            int, void *, void *, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace mxg
