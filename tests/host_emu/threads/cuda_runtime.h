/* Host stand-in for the CUDA runtime names the CUDA-core kernels use, for the
 * threaded race check: every CUDA thread of a CTA is a host thread, and
 * __syncthreads() is a std::barrier over the CTA's threads, so ThreadSanitizer
 * sees exactly the happens-before edges the barriers give on the device. */
#pragma once
#include <algorithm>
#include <atomic>
#include <barrier>
#include <cmath>
#include <cstdint>
#include <cstring>
using std::max;
using std::min;
typedef void *cudaStream_t;
struct host_uint3 { unsigned x, y, z; };
extern thread_local host_uint3 threadIdx, blockIdx, gridDim;
extern std::barrier<> *host_cta_barrier;
#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __shared__
#define __syncthreads() (host_cta_barrier->arrive_and_wait())
inline float atomicAdd(float *a, float v)
{
    return std::atomic_ref<float>(*a).fetch_add(v);
}
