// Per-device status word written by kernels whose bounded waits run out.
#include "gdn.h"
#include "gdn_status.cuh"

namespace gdn {

int read_and_clear_device_status(cudaStream_t stream)
{
    int host = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&host, g_device_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    return host == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

}  // namespace gdn
