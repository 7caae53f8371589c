// gdr_tc.cu -- tensor-core (tcgen05) kernel; placeholder until it lands.
#include "gdr_internal.h"

namespace gdr {
__device__ int g_device_status = 0;

int read_and_clear_device_status()
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return -1;
    return v;
}

bool tc_supports(const Params &) { return false; }
int launch_tc(const Params &, cudaStream_t) { return 5; }
}  // namespace gdr
