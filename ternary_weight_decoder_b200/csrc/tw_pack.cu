// tw_pack.cu — per-tensor ternarisation (s = 1/mean|W|) and 2-bit packing,
// plus the debug unpacker.
//
// Method: "VibeVoice-ASR-BitNet-ONNX" model page, "Quantization" table, row
// "LM projections (196 mats)": I2_S ternary weights with a per-tensor scale
// s = 1/mean|W|; codes are -1, 0 or +1 ("The Paper Says ARM Support" post,
// "What the model is trying to do").  mean|W| is accumulated in fp64 in a
// fixed order (each row over k, then the rows over n) so that the codes do
// not depend on how the sum is scheduled: one thread per row adds its row
// in k order, one thread adds the row sums in n order.  Both stage their
// operands through shared memory with coalesced loads, so that only the
// chains of dependent fp64 additions remain serial.
#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr double kMeanFloor = 1e-5;

constexpr int kRowsPerBlock = 128;   // one thread per row; 4 warps
constexpr int kSumChunk = 32;        // k per staged chunk (K is a multiple of 128)

// Rows n0 .. n0 + 127 of the block: per chunk of 32 k, warp w loads rows
// 32w .. 32w + 31 with one coalesced 128-byte load each (lane = k), then
// thread t adds row t's 32 values in k order.
__global__ void __launch_bounds__(kRowsPerBlock) k_row_abs_sum(const float *__restrict__ W, int64_t N,
                                                               int64_t K, double *__restrict__ rowsum,
                                                               uint32_t *err)
{
    __shared__ float tile[kRowsPerBlock][kSumChunk + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * kRowsPerBlock;
    const int64_t n = n0 + threadIdx.x;
    double s = 0.0;
    bool finite = true;
    for (int64_t k0 = 0; k0 < K; k0 += kSumChunk) {
        float v[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            const int64_t row = n0 + 32 * warp + r;
            v[r] = row < N ? __ldg(W + row * K + k0 + lane) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < 32; ++r)
            tile[32 * warp + r][lane] = v[r];
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kSumChunk; ++j) {
            const float x = tile[threadIdx.x][j];
            finite &= isfinite(x);
            s = __dadd_rn(s, fabs((double)x));
        }
        __syncthreads();
    }
    if (n < N) {
        rowsum[n] = s;
        if (!finite)
            atomicOr(err, EFLAG_NONFINITE);
    }
}

// ws layout: [0] double s = 1/mean; [32..] row sums.
constexpr int kTotalThreads = 256;
constexpr int kTotalChunk = 2048;    // row sums staged per step (16 KB)

// The block stages the row sums through shared memory; thread 0 adds them
// in n order.
__global__ void __launch_bounds__(kTotalThreads) k_total(const double *__restrict__ rowsum, int64_t N,
                                                         int64_t K, double *s_out, double *mean_abs,
                                                         float *wscale)
{
    __shared__ double buf[kTotalChunk];
    double t = 0.0;
    for (int64_t n0 = 0; n0 < N; n0 += kTotalChunk) {
        const int cnt = (int)(N - n0 < kTotalChunk ? N - n0 : kTotalChunk);
        for (int i = threadIdx.x; i < cnt; i += kTotalThreads)
            buf[i] = rowsum[n0 + i];
        __syncthreads();
        if (threadIdx.x == 0)
            for (int i = 0; i < cnt; ++i)
                t = __dadd_rn(t, buf[i]);
        __syncthreads();
    }
    if (threadIdx.x != 0)
        return;
    double mean = __ddiv_rn(t, (double)(N * K));
    if (!(mean >= kMeanFloor))
        mean = kMeanFloor;
    *s_out = __ddiv_rn(1.0, mean);
    if (mean_abs)
        *mean_abs = mean;
    *wscale = __double2float_rn(mean);
}

// One thread per packed 32-bit word.  Word w of the matrix: tile w/128
// (row block rb = tile / KT, k tile kt = tile % KT); inside the tile word
// wi = w % 128 = 4*lane + j with lane = 4*g + t; it holds row
// 16*rb + g + 8*(j&1), k = 128*kt + 64*(j>>1) + 16*t + 4*s + b at bit 8b+2s.
__global__ void k_pack(const float *__restrict__ W, int64_t N, int64_t K,
                       const double *__restrict__ s_ptr, uint32_t *__restrict__ packed,
                       int64_t n_words)
{
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= n_words)
        return;
    const int64_t KT = K / kTileK;
    const int64_t tile = w >> 7;
    const int wi = (int)(w & 127);
    const int lane = wi >> 2, j = wi & 3;
    const int g = lane >> 2, t = lane & 3;
    const int64_t rb = tile / KT, kt = tile - rb * KT;
    const int64_t row = rb * kTileRows + g + 8 * (j & 1);
    const int64_t k0 = kt * kTileK + 64 * (j >> 1) + 16 * t;
    uint32_t word = 0x55555555u;  // code 0 everywhere (padding rows)
    if (row < N) {
        const double s = *s_ptr;
        const float4 *src = reinterpret_cast<const float4 *>(W + row * K + k0);
        float v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = __ldg(src + q);
            v[4 * q + 0] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
        word = 0;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            double r = rint(__dmul_rn((double)v[kk], s));
            r = fmin(fmax(r, -1.0), 1.0);
            const uint32_t c = (uint32_t)((int)r + 1);
            const int sft = kk >> 2, b = kk & 3;
            word |= c << (8 * b + 2 * sft);
        }
    }
    packed[w] = word;
}

// One thread per packed word: write its 16 codes as int8 (row-major) and
// count fields holding the invalid pattern 3.
__global__ void k_unpack(const uint32_t *__restrict__ packed, int64_t N, int64_t K,
                         int8_t *__restrict__ codes, int32_t *invalid_count, int64_t n_words)
{
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= n_words)
        return;
    const int64_t KT = K / kTileK;
    const int64_t tile = w >> 7;
    const int wi = (int)(w & 127);
    const int lane = wi >> 2, j = wi & 3;
    const int g = lane >> 2, t = lane & 3;
    const int64_t rb = tile / KT, kt = tile - rb * KT;
    const int64_t row = rb * kTileRows + g + 8 * (j & 1);
    const int64_t k0 = kt * kTileK + 64 * (j >> 1) + 16 * t;
    const uint32_t word = packed[w];
    int bad = 0;
    uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
        const int sft = kk >> 2, b = kk & 3;
        const uint32_t f = (word >> (8 * b + 2 * sft)) & 3u;
        bad += (f == 3u);
        const int c = (f == 3u) ? 0 : (int)f - 1;
        out[kk >> 2] |= ((uint32_t)(uint8_t)(int8_t)c) << (8 * (kk & 3));
    }
    if (row < N)
        *reinterpret_cast<uint4 *>(codes + row * K + k0) = make_uint4(out[0], out[1], out[2], out[3]);
    if (bad && invalid_count)
        atomicAdd(invalid_count, bad);
}

}  // namespace

cudaError_t launch_ternarize(const float *W, int64_t N, int64_t K, uint8_t *packed,
                             double *mean_abs, float *wscale, void *ws, uint32_t *err,
                             cudaStream_t stream)
{
    double *s_ptr = reinterpret_cast<double *>(ws);
    double *rowsum = reinterpret_cast<double *>(static_cast<char *>(ws) + 256);
    k_row_abs_sum<<<(unsigned)ceil_div(N, kRowsPerBlock), kRowsPerBlock, 0, stream>>>(W, N, K, rowsum,
                                                                                      err);
    k_total<<<1, kTotalThreads, 0, stream>>>(rowsum, N, K, s_ptr, mean_abs, wscale);
    const int64_t n_words = ceil_div(N, kTileRows) * kTileRows * K / 16;
    k_pack<<<(unsigned)ceil_div(n_words, 256), 256, 0, stream>>>(
        W, N, K, s_ptr, reinterpret_cast<uint32_t *>(packed), n_words);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes,
                          int32_t *invalid_count, cudaStream_t stream)
{
    const int64_t n_words = ceil_div(N, kTileRows) * kTileRows * K / 16;
    k_unpack<<<(unsigned)ceil_div(n_words, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(packed), N, K, codes, invalid_count, n_words);
    return cudaGetLastError();
}

}  // namespace tw
