// gdr_epilogue.cu -- the readout epilogue of the SLA recurrence ("Systolic Linear
// Attention: Co-Designing Tile-Grouped Gated Delta Attention for TPUs", §2.3
// Eq. (5)): o_{t,m} <- sigmoid(z_{t,m}) * RMSNorm(o_{t,m}) per (token, value head)
// row of dv channels, in place on the output of gdr_chunk_fwd.
//
// Memory-bound (o and z read once, o written once), so the main kernel moves 16
// bytes a load: a lane holds 8 consecutive channels, a row takes the next power
// of two of dv / 8 lanes (16 at dv = 128: two rows a warp), the sum of squares is
// a shuffle reduction over those lanes in fp32, and warps stride over the rows on
// a grid sized to the SMs.  Rows whose dv is not a multiple of 8, or unaligned
// buffers, take the plain kernel: one warp per row, lane l on channels l, l + 32.
#include <cuda_bf16.h>

#include "gdr.h"
#include "gdr_internal.h"

namespace {

constexpr int kWarps = 8;
constexpr int kMaxPerLane = 8;   // dv <= 256

template <bool BF>
__device__ __forceinline__ float ld(const void *p, long i)
{
    if constexpr (BF)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else
        return static_cast<const float *>(p)[i];
}

template <bool BF>
__device__ __forceinline__ void st(void *p, long i, float v)
{
    if constexpr (BF)
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
    else
        static_cast<float *>(p)[i] = v;
}

// 8 channels at element offset i (16-byte aligned for bf16, 32 for fp32)
template <bool BF>
__device__ __forceinline__ void ld8(const void *p, long i, float *v)
{
    if constexpr (BF) {
        const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
        const float4 b = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

template <bool BF>
__device__ __forceinline__ void st8(void *p, long i, const float *v)
{
    if constexpr (BF) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p) + i) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(p) + i) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(static_cast<float *>(p) + i + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// LPR lanes per row (a power of two, 8 LPR >= dv), 32 / LPR rows per warp pass
template <bool BF, int LPR>
__global__ void __launch_bounds__(kWarps * 32)
out_gate_rmsnorm_vec_kernel(void *o, const void *z, const float *w, float eps, long rows, int dv)
{
    constexpr int RPW = 32 / LPR;
    const int lane = threadIdx.x & 31, sub = lane / LPR, c = 8 * (lane % LPR);
    const long wid = (long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long stride = (long)gridDim.x * kWarps * RPW;
    float wt[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        wt[e] = (w != nullptr && c + e < dv) ? w[c + e] : 1.f;
    for (long row0 = wid * RPW; row0 < rows; row0 += stride) {
        const long row = row0 + sub;
        const bool live = row < rows && c < dv;
        const long base = row * dv + c;
        float x[8], g[8];
        float ss = 0.f;
        if (live) {
            ld8<BF>(o, base, x);
            ld8<BF>(z, base, g);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                ss += x[e] * x[e];
        }
#pragma unroll
        for (int d = LPR / 2; d > 0; d >>= 1)
            ss += __shfl_xor_sync(0xffffffffu, ss, d);
        if (live) {
            const float inv = rsqrtf(ss / (float)dv + eps);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                x[e] = x[e] * inv * wt[e] / (1.f + __expf(-g[e]));
            st8<BF>(o, base, x);
        }
    }
}

template <bool BF>
__global__ void __launch_bounds__(kWarps * 32)
out_gate_rmsnorm_kernel(void *o, const void *z, const float *w, float eps, long rows, int dv)
{
    const long row = (long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows)
        return;
    const long base = row * dv;
    float x[kMaxPerLane];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxPerLane; ++u) {
        const int i = lane + 32 * u;
        x[u] = i < dv ? ld<BF>(o, base + i) : 0.f;
        ss += x[u] * x[u];
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1)
        ss += __shfl_xor_sync(0xffffffffu, ss, d);
    const float inv = rsqrtf(ss / (float)dv + eps);
#pragma unroll
    for (int u = 0; u < kMaxPerLane; ++u) {
        const int i = lane + 32 * u;
        if (i < dv) {
            const float gate = 1.f / (1.f + __expf(-ld<BF>(z, base + i)));
            st<BF>(o, base + i, gate * x[u] * inv * (w != nullptr ? w[i] : 1.f));
        }
    }
}

}  // namespace

extern "C" gdr_status gdr_output_gate_rmsnorm(const gdr_shape *shape, void *o, const void *z,
                                              const float *weight, float eps, void *stream)
{
    if (shape == nullptr || !(eps >= 0.f) || eps > 1e30f)
        return GDR_ERR_ARG;
    if (shape->out_dtype != GDR_F32 && shape->out_dtype != GDR_BF16)
        return GDR_ERR_DTYPE;
    if (shape->B < 0 || shape->T < 0 || shape->Hv < 1 || shape->dv < 1 || shape->dv > 256)
        return GDR_ERR_SHAPE;
    const long rows = (long)shape->B * shape->Hv * shape->T;
    if (rows == 0)
        return GDR_OK;
    if (o == nullptr || z == nullptr)
        return GDR_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf = shape->out_dtype == GDR_BF16;
    const int dv = shape->dv;
    const uintptr_t al = bf ? 15u : 31u;
    if (dv % 8 == 0 && ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(z)) & al) == 0) {
        int lpr = 1;
        while (8 * lpr < dv)
            lpr *= 2;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const long per_block = (long)kWarps * (32 / lpr);
        const long want = (rows + per_block - 1) / per_block;
        const unsigned grid = (unsigned)(want < 8L * sms ? want : 8L * sms);
#define GDR_EPI_LAUNCH(L)                                                                          \
    (bf ? (out_gate_rmsnorm_vec_kernel<true, L><<<grid, kWarps * 32, 0, s>>>(o, z, weight, eps, rows, dv)) \
        : (out_gate_rmsnorm_vec_kernel<false, L><<<grid, kWarps * 32, 0, s>>>(o, z, weight, eps, rows, dv)))
        switch (lpr) {
        case 1: GDR_EPI_LAUNCH(1); break;
        case 2: GDR_EPI_LAUNCH(2); break;
        case 4: GDR_EPI_LAUNCH(4); break;
        case 8: GDR_EPI_LAUNCH(8); break;
        case 16: GDR_EPI_LAUNCH(16); break;
        default: GDR_EPI_LAUNCH(32); break;
        }
#undef GDR_EPI_LAUNCH
        return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
    }
    const long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffL)
        return GDR_ERR_SHAPE;
    if (bf)
        out_gate_rmsnorm_kernel<true><<<(unsigned)blocks, kWarps * 32, 0, s>>>(o, z, weight, eps, rows,
                                                                             shape->dv);
    else
        out_gate_rmsnorm_kernel<false><<<(unsigned)blocks, kWarps * 32, 0, s>>>(o, z, weight, eps, rows,
                                                                              shape->dv);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}
