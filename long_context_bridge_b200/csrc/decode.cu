// decode.cu -- placeholder until the decode kernels land
#include "common.cuh"
#include "kernels.h"
namespace hs2 {

HS2_STATUS_ACCESSOR(status_decode)

size_t decode_workspace_bytes(int, int64_t, int, int, int, int) { return 0; }
cudaError_t launch_decode(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace hs2
