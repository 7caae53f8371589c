/* Host stand-in for the few CUDA runtime names that gdr_simt.cu's kernel uses,
 * so that its source compiles as plain C++ for the host-emulation test: one
 * thread per CTA, CTAs run one after another, __syncthreads() is a no-op (with
 * a single thread every phase completes before the next begins). */
#pragma once
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
using std::max;
using std::min;
typedef void *cudaStream_t;
struct host_uint3 { unsigned x, y, z; };
extern thread_local host_uint3 threadIdx, blockIdx, gridDim;
#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __shared__
#define __syncthreads() ((void)0)
/* one thread at a time: an atomic add is a plain add */
inline float atomicAdd(float *a, float v)
{
    const float old = *a;
    *a = old + v;
    return old;
}
