// Tensor-core (tcgen05 / TMEM / TMA) chunked GDN forward for sm_100a.
#include "gdn_common.cuh"
#include "gdn_status.cuh"


namespace gdn {

bool tc_supported(int dk, int dv, int chunk_len)
{
    (void)dk; (void)dv; (void)chunk_len;
    return false;
}

cudaError_t launch_tc(const FwdParams& p, int chunk_len, cudaStream_t stream)
{
    (void)p; (void)chunk_len; (void)stream;
    return cudaErrorNotSupported;
}

}  // namespace gdn
