// tw_tp.cu — the pieces of a tensor-parallel split of the ternary
// projections across ranks, each rank one GPU (Megatron-style pairing):
//
//   column-parallel (q, k, v, gate, up): rank r holds a slice of the weight
//     rows and the whole input; its output is its slice of y.  Nothing is
//     exchanged.
//   row-parallel (o, down): rank r holds a slice of the input channels k and
//     the matching columns of every weight row.  The per-token scale of the
//     activations must be that of the whole row, so the ranks first take the
//     maximum of their row maxima (a max all-reduce of M floats); each then
//     quantises its slice with that scale, forms its partial integer sums,
//     and the ranks add those (an int32 sum all-reduce of M x N) before the
//     rescale.  Integer addition is exact and order-free, so every rank ends
//     with the bytes one GPU would have produced.
//
// Here: slicing packed codes (the per-tensor scale stays that of the whole
// matrix, computed before the split), row maxima, quantisation with a given
// scale, and the rescale of summed accumulators.  The collectives run in
// the caller (NCCL through torch.distributed).  The partial sums come from
// tw_ternary_linear_q.
//
// The pages describe single-process CPU inference; the split is this
// library's own, and its result is defined to be the single-device result.
#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kThreadsTp = 256;
constexpr uint32_t kZeroCodes = 0x55555555u;   // sixteen codes 0 (stored as 1 in two bits)

// One thread per 32-bit word of the slice.  Tile (rb, kt) of the slice is
// tile (rb + rb0, kt + kt0) of the source; rows at or past `rows` (only in
// the slice's last row block) are written as code 0.
__global__ void k_pack_slice(const uint32_t *__restrict__ src, int64_t kt_src,
                             uint32_t *__restrict__ dst, int64_t kt_out, int64_t words,
                             int64_t rb0, int64_t kt0, int64_t rows)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t w = i & 127, tile = i >> 7;
        const int64_t kt = tile % kt_out, rb = tile / kt_out;
        const int l = (int)(w >> 2), j = (int)(w & 3);
        const int64_t row = rb * kTileRows + (l >> 2) + 8 * (j & 1);
        dst[i] = row < rows ? __ldg(src + ((rb + rb0) * kt_src + kt + kt0) * 128 + w) : kZeroCodes;
    }
}

// max |x| of each row (exact; one block per row).
__global__ void __launch_bounds__(kThreadsTp) k_row_absmax(const float *__restrict__ x, int64_t K,
                                                            float *__restrict__ amax)
{
    __shared__ float red[kThreadsTp / 32];
    const float4 *row = reinterpret_cast<const float4 *>(x + (int64_t)blockIdx.x * K);
    float a = 0.f;
    for (int64_t i = threadIdx.x; i < K / 4; i += kThreadsTp) {
        const float4 v = __ldg(row + i);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreadsTp / 32; ++w)
            a = fmaxf(a, red[w]);
        amax[blockIdx.x] = fmaxf(a, red[0]);
    }
}

// q = clamp(rint(x * (127 / amax[m])), -128, 127) with the given row scale
// (fp32 multiply, IEEE division, half to even); amax == 0 gives q == 0;
// qsum[m] = sum of the row's q.  One block per row.
__global__ void __launch_bounds__(kThreadsTp) k_quantize_given(const float *__restrict__ x, int64_t K,
                                                                const float *__restrict__ amax,
                                                                int8_t *__restrict__ xq,
                                                                int32_t *__restrict__ qsum)
{
    __shared__ int red[kThreadsTp / 32];
    const int64_t m = blockIdx.x;
    const float4 *row = reinterpret_cast<const float4 *>(x + m * K);
    uint32_t *qrow = reinterpret_cast<uint32_t *>(xq + m * K);
    const float a = __ldg(amax + m);
    const bool zero = a == 0.f;
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    int sum = 0;
    for (int64_t i = threadIdx.x; i < K / 4; i += kThreadsTp) {
        const float4 v = __ldg(row + i);
        int q[4] = {0, 0, 0, 0};
        if (!zero) {
            q[0] = min(max(__float2int_rn(__fmul_rn(v.x, scale)), -128), 127);
            q[1] = min(max(__float2int_rn(__fmul_rn(v.y, scale)), -128), 127);
            q[2] = min(max(__float2int_rn(__fmul_rn(v.z, scale)), -128), 127);
            q[3] = min(max(__float2int_rn(__fmul_rn(v.w, scale)), -128), 127);
        }
        sum += q[0] + q[1] + q[2] + q[3];
        qrow[i] = (uint32_t)(q[0] & 0xff) | ((uint32_t)(q[1] & 0xff) << 8) |
                  ((uint32_t)(q[2] & 0xff) << 16) | ((uint32_t)(q[3] & 0xff) << 24);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0 && qsum) {
        int s = 0;
        for (int w = 0; w < kThreadsTp / 32; ++w)
            s += red[w];
        qsum[m] = s;
    }
}

// y = ((float)acc * (amax[m] / 127)) * wscale, the rounding of every
// projection epilogue of this library.
__global__ void k_rescale_acc(const int32_t *__restrict__ acc, int64_t M, int64_t N,
                              const float *__restrict__ amax, const float *__restrict__ wscale,
                              float *__restrict__ y)
{
    const float ws = __ldg(wscale);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < M * N;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float sa = __fdiv_rn(__ldg(amax + i / N), 127.f);
        y[i] = __fmul_rn(__fmul_rn((float)__ldg(acc + i), sa), ws);
    }
}

unsigned grid_for(int64_t n)
{
    const int64_t b = (n + kThreadsTp - 1) / kThreadsTp;
    return (unsigned)(b < 1 ? 1 : b > 148 * 16 ? 148 * 16 : b);
}

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int fail_cuda(cudaError_t e) { return record_error(TW_ERR_CUDA, cudaGetErrorString(e)); }

}  // namespace
}  // namespace tw

extern "C" {

TW_API int tw_pack_slice(const void *packed, int64_t N, int64_t K, int64_t n0, int64_t rows,
                         int64_t k0, int64_t cols, void *out, size_t out_bytes, tw_stream_t stream)
{
    tw::clear_error();
    if (!packed || !out)
        return tw::record_error(TW_ERR_NULL, "tw_pack_slice: packed and out are required");
    if (N < 1 || K < 1 || K % tw::kTileK || rows < 1 || cols < 1 || n0 < 0 || k0 < 0 ||
        n0 % tw::kTileRows || k0 % tw::kTileK || cols % tw::kTileK || n0 + rows > N ||
        k0 + cols > K)
        return tw::record_error(TW_ERR_SHAPE, "tw_pack_slice: the slice must lie inside [N x K], "
                                "start at a multiple of 16 rows and 128 columns, and span a "
                                "multiple of 128 columns");
    if (!tw::a16(packed) || !tw::a16(out))
        return tw::record_error(TW_ERR_ALIGN, "tw_pack_slice: pointers must be 16-byte aligned");
    if (out_bytes < tw_packed_bytes(rows, cols))
        return tw::record_error(TW_ERR_BUFSIZE, "tw_pack_slice: out smaller than "
                                "tw_packed_bytes(rows, cols)");
    const int64_t kt_out = cols / tw::kTileK;
    const int64_t words = tw::ceil_div(rows, tw::kTileRows) * kt_out * 128;
    tw::k_pack_slice<<<tw::grid_for(words), tw::kThreadsTp, 0, stream>>>(
        static_cast<const uint32_t *>(packed), K / tw::kTileK, static_cast<uint32_t *>(out), kt_out,
        words, n0 / tw::kTileRows, k0 / tw::kTileK, rows);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TW_OK : tw::fail_cuda(e);
}

TW_API int tw_row_absmax(const float *x, int64_t M, int64_t K, float *amax, tw_stream_t stream)
{
    tw::clear_error();
    if (!x || !amax)
        return tw::record_error(TW_ERR_NULL, "tw_row_absmax: x and amax are required");
    if (M < 1 || K < 1 || K % 4 || M > (1 << 24) || K > (1 << 24))
        return tw::record_error(TW_ERR_SHAPE, "tw_row_absmax: need M >= 1 and K a positive multiple of 4");
    if (!tw::a16(x) || !tw::a16(amax))
        return tw::record_error(TW_ERR_ALIGN, "tw_row_absmax: pointers must be 16-byte aligned");
    tw::k_row_absmax<<<(unsigned)M, tw::kThreadsTp, 0, stream>>>(x, K, amax);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TW_OK : tw::fail_cuda(e);
}

TW_API int tw_quantize_act_given(const float *x, int64_t M, int64_t K, const float *amax, int8_t *xq,
                                 int32_t *qsum, tw_stream_t stream)
{
    tw::clear_error();
    if (!x || !amax || !xq)
        return tw::record_error(TW_ERR_NULL, "tw_quantize_act_given: x, amax and xq are required");
    if (M < 1 || K < 1 || K % 4 || M > (1 << 24) || K > (1 << 24))
        return tw::record_error(TW_ERR_SHAPE, "tw_quantize_act_given: need M >= 1 and K a positive "
                                "multiple of 4");
    if (!tw::a16(x) || !tw::a16(amax) || !tw::a16(xq) || (qsum && !tw::a16(qsum)))
        return tw::record_error(TW_ERR_ALIGN, "tw_quantize_act_given: pointers must be 16-byte aligned");
    tw::k_quantize_given<<<(unsigned)M, tw::kThreadsTp, 0, stream>>>(x, K, amax, xq, qsum);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TW_OK : tw::fail_cuda(e);
}

TW_API int tw_rescale_acc(const int32_t *acc, int64_t M, int64_t N, const float *amax,
                          const float *wscale, float *y, tw_stream_t stream)
{
    tw::clear_error();
    if (!acc || !amax || !wscale || !y)
        return tw::record_error(TW_ERR_NULL, "tw_rescale_acc: acc, amax, wscale and y are required");
    if (M < 1 || N < 1 || M > (1 << 24) || N > (1 << 24))
        return tw::record_error(TW_ERR_SHAPE, "tw_rescale_acc: need M, N >= 1");
    if (!tw::a16(acc) || !tw::a16(amax) || !tw::a16(wscale) || !tw::a16(y))
        return tw::record_error(TW_ERR_ALIGN, "tw_rescale_acc: pointers must be 16-byte aligned");
    tw::k_rescale_acc<<<tw::grid_for(M * N), tw::kThreadsTp, 0, stream>>>(acc, M, N, amax, wscale, y);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TW_OK : tw::fail_cuda(e);
}

}  // extern "C"
