// tw_quant.cu — stand-alone per-token int8 activation quantisation by absmax
// (the input of the prefill path and of the I8_S layer): one warp per row
// for rows of up to 1024 elements, one block per row above.  The decode path
// fuses the same arithmetic into its own kernel.
//
// amax = max|x| (exact), scale = 127.0f / amax (IEEE fp32 division),
// q = clamp(rint(x * scale), -128, 127) with one fp32 multiply and
// round-half-to-even; amax == 0 gives q = 0.  The pages name "fused INT8"
// operations only (xujun.org article, heterogeneous-quantisation section;
// aitrends summary, technical features); this is the plainest absmax reading.
#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kQThreads = 256;

__device__ __forceinline__ uint32_t quant4(float4 v, float scale, bool zero, int &sum)
{
    int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
    if (!zero) {
        q0 = min(max(__float2int_rn(__fmul_rn(v.x, scale)), -128), 127);
        q1 = min(max(__float2int_rn(__fmul_rn(v.y, scale)), -128), 127);
        q2 = min(max(__float2int_rn(__fmul_rn(v.z, scale)), -128), 127);
        q3 = min(max(__float2int_rn(__fmul_rn(v.w, scale)), -128), 127);
    }
    sum += q0 + q1 + q2 + q3;
    return (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
           ((uint32_t)(q3 & 0xff) << 24);
}

// One block per token row.
__global__ void __launch_bounds__(kQThreads) k_quantize(const float *__restrict__ x, int64_t K,
                                                        int8_t *__restrict__ xq,
                                                        float *__restrict__ amax_out,
                                                        int32_t *__restrict__ qsum_out)
{
    __shared__ float red_f[kQThreads / 32];
    __shared__ int red_i[kQThreads / 32];
    const int64_t m = blockIdx.x;
    const float4 *row = reinterpret_cast<const float4 *>(x + m * K);
    uint32_t *qrow = reinterpret_cast<uint32_t *>(xq + m * K);
    const int64_t K4 = K / 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    float a = 0.f;
    for (int64_t i = tid; i < K4; i += kQThreads) {
        const float4 v = __ldg(row + i);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0)
        red_f[warp] = a;
    __syncthreads();
    a = red_f[0];
#pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w)
        a = fmaxf(a, red_f[w]);

    const bool zero = (a == 0.f);
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    int sum = 0;
    for (int64_t i = tid; i < K4; i += kQThreads)
        qrow[i] = quant4(__ldg(row + i), scale, zero, sum);
#pragma unroll
    for (int o = 16; o; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0)
        red_i[warp] = sum;
    __syncthreads();
    if (tid == 0) {
        int s = 0;
        for (int w = 0; w < kQThreads / 32; ++w)
            s += red_i[w];
        amax_out[m] = a;
        if (qsum_out)
            qsum_out[m] = s;
    }
}

// One warp per token row, the row held in registers (K <= 32 * 4 * kWarpRegs):
// for short rows a block per row would leave most of its threads idle.
constexpr int kWarpRegs = 8;   // float4 per lane
__global__ void __launch_bounds__(kQThreads) k_quantize_warp(const float *__restrict__ x, int64_t M,
                                                             int64_t K, int8_t *__restrict__ xq,
                                                             float *__restrict__ amax_out,
                                                             int32_t *__restrict__ qsum_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t m = (int64_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
    if (m >= M)
        return;   // (whole warps)
    const float4 *row = reinterpret_cast<const float4 *>(x + m * K);
    uint32_t *qrow = reinterpret_cast<uint32_t *>(xq + m * K);
    const int K4 = (int)(K / 4);
    float4 v[kWarpRegs];
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < kWarpRegs; ++i) {
        const int idx = lane + 32 * i;
        v[i] = idx < K4 ? __ldg(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const bool zero = (a == 0.f);
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kWarpRegs; ++i) {
        const int idx = lane + 32 * i;
        if (idx < K4)
            qrow[idx] = quant4(v[i], scale, zero, sum);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        amax_out[m] = a;
        if (qsum_out)
            qsum_out[m] = sum;
    }
}

}  // namespace

cudaError_t launch_quantize(const float *x, int64_t M, int64_t K, int8_t *xq, float *amax,
                            int32_t *qsum, cudaStream_t stream)
{
    if (K <= 32 * 4 * kWarpRegs) {
        const int64_t rows_per_block = kQThreads / 32;
        k_quantize_warp<<<(unsigned)((M + rows_per_block - 1) / rows_per_block), kQThreads, 0, stream>>>(
            x, M, K, xq, amax, qsum);
    } else {
        k_quantize<<<(unsigned)M, kQThreads, 0, stream>>>(x, K, xq, amax, qsum);
    }
    return cudaGetLastError();
}

}  // namespace tw
