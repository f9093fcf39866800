// tw_decode.cu — fused activation-quantisation + ternary GEMV for decode
// (M <= 32 tokens), as one persistent launch over any number of projections.
//
// What it computes, per projection: q = absmax int8 quantisation of each
// token row of x, acc = q * codes^T in exact integer arithmetic, and
// y = ((float)acc * (amax/127)) * mean|W|.  (Per-tensor ternary weights with
// s = 1/mean|W|: "VibeVoice-ASR-BitNet-ONNX" model page, Quantization table;
// the weights of all 196 projections are read once per token, which is what
// bounds decode: "The Paper Says ARM Support" post, "What the model is
// trying to do".)
//
// Structure (one CTA per SM, 9 warps):
//   * The grid splits the concatenated 16-row blocks of all projections into
//     equal shares of packed bytes; each CTA streams its share once.
//   * Warp 8 (activation warp) quantises, for every projection the CTA
//     touches, the token rows of x into an int8 shared-memory buffer (double
//     buffered when it fits) together with amax/127 and sum(q) per token.
//   * Warps 0..7 (consumer warps) each own every 8th row block of the share.
//     Each keeps a private ring of 4 KB slots filled by 1-D bulk copies (the
//     TMA engine) that it issues itself, several chunks ahead, so the packed
//     codes stream from HBM independently of the arithmetic.
//   * Codes are decoded in registers: (word >> 2s) & 0x03030303 gives four
//     codes + 1 as bytes, which are fed straight into m16n8k32 int8 MMAs
//     (weights are the 16-row side, tokens the 8-column side).  The +1
//     offset is removed at the end with the per-token sum(q):
//     sum (c+1) q - sum q = sum c q, exactly.
//   * Every wait is bounded; a timeout sets the device error word, stops the
//     block and drains the copies still in flight before the block exits.
#include <cstring>

#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kNC = 8;                      // consumer warps
constexpr int kThreads = (kNC + 1) * 32;    // + activation warp
constexpr int kCT = 8;                      // tiles per ring chunk
constexpr int kChunk = kCT * kTileBytes;    // 4 KB
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMiscBytes = 2048;            // barriers, token info, plan
constexpr uint64_t kDrainNs = 1000000000ull;

struct DecodeParams {
    const DescRecord *table;  // null: use `single`
    DescRecord single;
    int count;
    int m0, mg;               // token group [m0, m0 + mg)
    int xb;                   // activation buffers (1 or 2)
    int xs;                   // activation row stride in shared memory
    int slots;                // ring slots per consumer warp
    int64_t total_rb, total_tiles;
    WaitCtl ctl;
};

struct Plan {
    int64_t rb_lo, rb_hi;
    int d_lo, d_hi;
    int abort_flag;
};

__device__ __forceinline__ const DescRecord &rec(const DecodeParams &p, int d)
{
    return p.table ? p.table[d] : p.single;
}

__device__ __forceinline__ int64_t rb_count(const DescRecord &r) { return (r.N + 15) >> 4; }

// First row block owned by CTA i of G: the first block whose first tile is
// at or after tile floor(total_tiles * i / G).
__device__ int64_t share_boundary(const DecodeParams &p, int i, int G)
{
    if (i <= 0)
        return 0;
    if (i >= G)
        return p.total_rb;
    const int64_t t = p.total_tiles * i / G;  // total_tiles < 2^40, i < 2^16
    int lo = 0, hi = p.count - 1;  // largest d with tile_begin <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rec(p, mid).tile_begin <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    const DescRecord &r = rec(p, lo);
    const int64_t KT = r.K / kTileK;
    const int64_t rl = (t - r.tile_begin + KT - 1) / KT;
    return r.rb_begin + rl;
}

__device__ int desc_of_rb(const DecodeParams &p, int64_t rb)
{
    int lo = 0, hi = p.count - 1;  // largest d with rb_begin <= rb
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rec(p, mid).rb_begin <= rb)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Walks the chunks of one consumer warp: every kNC-th row block of the CTA
// share, each cut into ceil(KT / kCT) chunks.
struct ChunkIter {
    int64_t rb, rb_end, rb_hi;
    int d, kc, nch, KT;
    bool valid;

    __device__ void load_desc(const DecodeParams &p)
    {
        const DescRecord &r = rec(p, d);
        rb_end = r.rb_begin + rb_count(r);
        KT = (int)(r.K / kTileK);
        nch = (KT + kCT - 1) / kCT;
    }
    __device__ void seek(const DecodeParams &p)
    {
        while (rb >= rb_end) {
            ++d;
            load_desc(p);
        }
    }
    __device__ void init(const DecodeParams &p, const Plan &pl, int w)
    {
        rb = pl.rb_lo + w;
        rb_hi = pl.rb_hi;
        kc = 0;
        valid = rb < rb_hi;
        if (valid) {
            d = pl.d_lo;
            load_desc(p);
            seek(p);
        }
    }
    __device__ void next(const DecodeParams &p)
    {
        if (++kc < nch)
            return;
        kc = 0;
        rb += kNC;
        valid = rb < rb_hi;
        if (valid)
            seek(p);
    }
};

__device__ __forceinline__ void issue_chunk(const DecodeParams &p, const ChunkIter &it,
                                            uint32_t dst, uint32_t bar)
{
    const DescRecord &r = rec(p, it.d);
    const int kt0 = it.kc * kCT;
    const int n = min(kCT, it.KT - kt0);
    const uint8_t *src =
        r.packed + ((it.rb - r.rb_begin) * (int64_t)it.KT + kt0) * (int64_t)kTileBytes;
    mbar_arrive_expect_tx(bar, (uint32_t)(n * kTileBytes));
    bulk_g2s(dst, src, (uint32_t)(n * kTileBytes), bar);
}

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

// Activation warp: quantise token rows [m0, m0+mg) of projection d into
// buffer b (row stride xs), amax/127 into sa[tok], sum(q) into qs[tok].
__device__ void quantise_rows(const DecodeParams &p, int d, uint8_t *xbuf, float *sa, int *qs,
                              int lane)
{
    const DescRecord &r = rec(p, d);
    const int64_t K = r.K, K4 = K / 4;
    for (int tok = 0; tok < p.mg; ++tok) {
        const float4 *row = reinterpret_cast<const float4 *>(r.x + (int64_t)(p.m0 + tok) * K);
        float a = 0.f;
#pragma unroll 4
        for (int64_t i = lane; i < K4; i += 32) {
            const float4 v = __ldg(row + i);
            a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const bool zero = (a == 0.f);
        const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
        uint32_t *dst = reinterpret_cast<uint32_t *>(xbuf + (int64_t)tok * p.xs);
        int sum = 0;
#pragma unroll 4
        for (int64_t i = lane; i < K4; i += 32)
            dst[i] = quant4(__ldg(row + i), scale, zero, sum);
#pragma unroll
        for (int o = 16; o; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            sa[tok] = __fdiv_rn(a, 127.f);
            qs[tok] = sum;
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_decode(const __grid_constant__ DecodeParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int ring_bytes = kNC * p.slots * kChunk;
    uint8_t *ring = smem;
    uint8_t *xbase = smem + ring_bytes;
    const int xbuf_bytes = p.mg * p.xs;
    uint8_t *misc = xbase + p.xb * xbuf_bytes;
    float *sa = reinterpret_cast<float *>(misc);             // [2][32]
    int *qs = reinterpret_cast<int *>(misc + 256);           // [2][32]
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc + 512);
    // bars: ring_full[kNC*slots], x_full[2], x_empty[2]
    Plan *plan = reinterpret_cast<Plan *>(misc + 512 + 8 * (kNC * p.slots + 4));
    const uint32_t bar_ring = smem_u32(bars);
    const uint32_t bar_xfull = bar_ring + 8 * kNC * p.slots;
    const uint32_t bar_xempty = bar_xfull + 16;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNC * p.slots; ++i)
            mbar_init(bar_ring + 8 * i, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_xfull + 8 * b, 32);
            mbar_init(bar_xempty + 8 * b, kNC * 32);
        }
        fence_barrier_init();
        const int G = gridDim.x, c = blockIdx.x;
        plan->rb_lo = share_boundary(p, c, G);
        plan->rb_hi = share_boundary(p, c + 1, G);
        plan->abort_flag = 0;
        if (plan->rb_lo < plan->rb_hi) {
            plan->d_lo = desc_of_rb(p, plan->rb_lo);
            plan->d_hi = desc_of_rb(p, plan->rb_hi - 1);
        } else {
            plan->d_lo = 0;
            plan->d_hi = -1;
        }
    }
    __syncthreads();
    const Plan pl = *plan;
    volatile int *abort_flag = &plan->abort_flag;

    if (warp == kNC) {
        // ------------------------------------------------ activation warp
        for (int d = pl.d_lo; d <= pl.d_hi; ++d) {
            const int seg = d - pl.d_lo, b = seg % p.xb;
            if (seg >= p.xb &&
                !mbar_wait(bar_xempty + 8 * b, ((seg / p.xb) - 1) & 1, p.ctl, abort_flag))
                return;
            quantise_rows(p, d, xbase + b * xbuf_bytes, sa + 32 * b, qs + 32 * b, lane);
            __syncwarp();
            mbar_arrive(bar_xfull + 8 * b);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int g = lane >> 2, t = lane & 3;
    const uint32_t ring_w = smem_u32(ring) + warp * p.slots * kChunk;
    const uint32_t bar_w = bar_ring + 8 * warp * p.slots;
    const uint32_t xbase_s = smem_u32(xbase);

    ChunkIter cons, prod;
    cons.init(p, pl, warp);
    prod = cons;
    int issued = 0, consumed = 0;
    if (lane == 0) {
        for (int s = 0; s < p.slots && prod.valid; ++s) {
            issue_chunk(p, prod, ring_w + s * kChunk, bar_w + 8 * s);
            prod.next(p);
            ++issued;
        }
    } else {
        for (int s = 0; s < p.slots && prod.valid; ++s) {
            prod.next(p);
            ++issued;
        }
    }

    bool ok = true;
    for (int d = pl.d_lo; d <= pl.d_hi && ok; ++d) {
        const int seg = d - pl.d_lo, b = seg % p.xb;
        if (!mbar_wait(bar_xfull + 8 * b, (seg / p.xb) & 1, p.ctl, abort_flag)) {
            ok = false;
            break;
        }
        const DescRecord &r = rec(p, d);
        const float wscale = __ldg(r.wscale);
        const uint32_t xrow = xbase_s + b * xbuf_bytes;

        while (cons.valid && cons.d == d) {
            int acc[2][NT][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        acc[h][nt][i] = 0;
            const int64_t rb = cons.rb;
            const int nch = cons.nch, KT = cons.KT;  // cons moves on after the last chunk
            for (int kc = 0; kc < nch; ++kc) {
                const int slot = consumed % p.slots;
                if (!mbar_wait(bar_w + 8 * slot, (consumed / p.slots) & 1, p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                const int kt0 = kc * kCT;
                const int n = min(kCT, KT - kt0);
                const uint32_t src = ring_w + slot * kChunk + lane * 16;
                for (int i = 0; i < n; ++i) {
                    const uint4 a = lds128(src + i * kTileBytes);
                    const uint32_t xk = xrow + (kt0 + i) * kTileK + 16 * t;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t w0 = h ? a.z : a.x;  // row g
                        const uint32_t w1 = h ? a.w : a.y;  // row g + 8
                        uint4 bx[NT];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int tok = 8 * nt + g;
                            bx[nt] = tok < p.mg ? lds128(xk + tok * p.xs + 64 * h)
                                                : make_uint4(0, 0, 0, 0);
                        }
                        const uint32_t m3 = 0x03030303u;
                        const uint32_t a00 = w0 & m3, a01 = w1 & m3;
                        const uint32_t a02 = (w0 >> 2) & m3, a03 = (w1 >> 2) & m3;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_s8_16832(acc[0][nt], a00, a01, a02, a03, bx[nt].x, bx[nt].y);
                        const uint32_t a10 = (w0 >> 4) & m3, a11 = (w1 >> 4) & m3;
                        const uint32_t a12 = (w0 >> 6) & m3, a13 = (w1 >> 6) & m3;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_s8_16832(acc[1][nt], a10, a11, a12, a13, bx[nt].z, bx[nt].w);
                    }
                }
                __syncwarp();
                ++consumed;
                if (prod.valid) {
                    if (lane == 0) {
                        fence_proxy_async_smem();
                        issue_chunk(p, prod, ring_w + slot * kChunk, bar_w + 8 * slot);
                    }
                    prod.next(p);
                    ++issued;
                }
                cons.next(p);
            }
            if (!ok)
                break;
            // epilogue of row block rb: rows 16*rl + g (+8), tokens 8nt + 2t (+1)
            const int64_t rl = rb - r.rb_begin;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = 8 * nt + 2 * t + (i & 1);
                    const int64_t row = rl * kTileRows + g + 8 * (i >> 1);
                    if (tok < p.mg && row < r.N) {
                        const int v = acc[0][nt][i] + acc[1][nt][i] - qs[32 * b + tok];
                        const int64_t o = (int64_t)(p.m0 + tok) * r.N + row;
                        r.y[o] = __fmul_rn(__fmul_rn((float)v, sa[32 * b + tok]), wscale);
                        if (r.acc_out)
                            r.acc_out[o] = v;
                    }
                }
            }
        }
        if (!ok)
            break;
        mbar_arrive(bar_xempty + 8 * b);
    }

    if (!ok) {
        // Drain: wait for every copy this warp still has in flight.
        WaitCtl drain = p.ctl;
        drain.timeout_ns = kDrainNs;
        for (int i = consumed; i < issued; ++i)
            mbar_wait(bar_w + 8 * (i % p.slots), (i / p.slots) & 1, drain, nullptr);
    }
}

__global__ void k_wait_probe(WaitCtl ctl)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait(b, 0, ctl, nullptr);  // nothing arrives: must time out
}

template <int NT>
cudaError_t launch_nt(const DecodeParams &p, int grid, int smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(k_decode<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess)
        return e;
    k_decode<NT><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch &L, uint32_t *err, uint64_t timeout_ns,
                          cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;

    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    if (L.single)
        p.single = *L.single;
    p.count = L.count;
    p.total_rb = L.total_rb;
    p.total_tiles = L.total_tiles;
    p.xs = (int)(L.max_K + 64);
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;

    // Shared-memory plan: ring, then 1 or 2 activation buffers of mg rows.
    const int M = (int)L.M;
    auto fits = [&](int s, int m, int b) {
        return 1024 + kNC * s * kChunk + b * m * p.xs + kMiscBytes <= kSmemLimit;
    };
    // Largest token group that fits with a ring of 4 (else 3, else 2)
    // slots per warp; a second activation buffer only when it also fits.
    int slots = 0, mg = M, xb = 1;
    while (true) {
        for (int s = 4; s >= 2 && !slots; --s)
            if (fits(s, mg, 1))
                slots = s;
        if (slots)
            break;
        if (mg == 1)
            return cudaErrorInvalidValue;
        mg = mg > 8 ? mg - 8 : mg - 1;
    }
    if (fits(slots, mg, 2))
        xb = 2;
    p.slots = slots;
    p.xb = xb;
    const int smem = 1024 + kNC * slots * kChunk + xb * mg * p.xs + kMiscBytes;
    int64_t grid64 = L.total_rb < sms ? L.total_rb : sms;
    const int grid = (int)(grid64 < 1 ? 1 : grid64);

    for (int m0 = 0; m0 < M; m0 += mg) {
        p.m0 = m0;
        p.mg = (M - m0) < mg ? (M - m0) : mg;
        const int nt = (p.mg + 7) / 8;
        switch (nt) {
        case 1: e = launch_nt<1>(p, grid, smem, stream); break;
        case 2: e = launch_nt<2>(p, grid, smem, stream); break;
        case 3: e = launch_nt<3>(p, grid, smem, stream); break;
        default: e = launch_nt<4>(p, grid, smem, stream); break;
        }
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

cudaError_t launch_wait_probe(uint32_t *err, uint64_t timeout_ns, cudaStream_t stream)
{
    WaitCtl ctl{err, timeout_ns};
    k_wait_probe<<<1, 32, 0, stream>>>(ctl);
    return cudaGetLastError();
}

}  // namespace tw
