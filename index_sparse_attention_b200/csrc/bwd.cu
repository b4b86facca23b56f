// bwd.cu -- placeholder until the backward kernels land.
#include "sa_device.cuh"
#include "sa_kernels.h"
namespace sa {
int launch_bwd(const AttnArgs&, const TensorMaps&, cudaStream_t) { return SA_ERR_UNSUPPORTED; }
}  // namespace sa
