// tw_chain.cu — the weight-free steps between the projections of the
// decoder-layer chain: identity attention over grouped KV heads, the
// single-precision residual add and SiLU(gate) * up.  (The decoder layer of
// the Qwen2.5-1.5B LM: "VibeVoice-ASR-BitNet-ONNX" model page, "Layout".)
// They move a few hundred KB per layer at most, so each is one grid-stride
// launch of at most one wave; the time that matters is the launch itself.
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kEwThreads = 256;
constexpr int64_t kEwMaxBlocks = 148 * 8;

unsigned ew_blocks(int64_t n)
{
    const int64_t b = ceil_div(n, kEwThreads);
    return (unsigned)(b < 1 ? 1 : b > kEwMaxBlocks ? kEwMaxBlocks : b);
}

// a[m, head * head_dim + c] = v[m, (head / group) * head_dim + c]: every token
// attends only to itself, so its attention output is its own v, each KV
// head serving the `group` query heads that share it.
__global__ void k_gqa_expand(const float *__restrict__ v, float *__restrict__ a, int64_t n,
                             int64_t kv_dim, int64_t hidden, int64_t head_dim, int64_t group)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / hidden, col = i - m * hidden;
        const int64_t head = col / head_dim, c = col - head * head_dim;
        a[i] = v[m * kv_dim + (head / group) * head_dim + c];
    }
}

__global__ void k_add_f32(const float *__restrict__ x, const float *__restrict__ y,
                          float *__restrict__ out, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __fadd_rn(x[i], y[i]);
}

// SiLU(g) * u with SiLU(z) = z / (1 + e^-z), each operation rounded once.
__global__ void k_silu_mul(const float *__restrict__ g, const float *__restrict__ u,
                           float *__restrict__ out, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float z = g[i];
        out[i] = __fmul_rn(__fdiv_rn(z, __fadd_rn(1.0f, expf(-z))), u[i]);
    }
}

}  // namespace

cudaError_t launch_gqa_expand(const float *v, float *a, int64_t M, int64_t kv_dim,
                              int64_t hidden, int64_t head_dim, cudaStream_t stream)
{
    const int64_t n = M * hidden;
    const int64_t group = (hidden / head_dim) / (kv_dim / head_dim);
    k_gqa_expand<<<ew_blocks(n), kEwThreads, 0, stream>>>(v, a, n, kv_dim, hidden, head_dim, group);
    return cudaGetLastError();
}

cudaError_t launch_add_f32(const float *x, const float *y, float *out, int64_t n,
                           cudaStream_t stream)
{
    k_add_f32<<<ew_blocks(n), kEwThreads, 0, stream>>>(x, y, out, n);
    return cudaGetLastError();
}

cudaError_t launch_silu_mul(const float *g, const float *u, float *out, int64_t n,
                            cudaStream_t stream)
{
    k_silu_mul<<<ew_blocks(n), kEwThreads, 0, stream>>>(g, u, out, n);
    return cudaGetLastError();
}

}  // namespace tw
