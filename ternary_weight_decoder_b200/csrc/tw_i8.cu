// tw_i8.cu — the I8_S linear layer: int8 weights with one absmax scale per
// tensor, int8 activations per token, int32 accumulation on the 5th-
// generation tensor cores, and bias + ReLU fused into the epilogue:
//   acc[m, n] = sum_k xq[m, k] * wq[n, k]                    (exact int32)
//   y[m, n]   = relu?(((float)acc * (amax_x[m]/127)) * (amax_w/127) + bias[n])
// (The audio encoder keeps int8 weights and activations and swaps GELU for
// ReLU: "VibeVoice-ASR-BitNet-ONNX" model page, "Quantization" table, row
// "VAE encoders"; its fused int8 routines join matmul, bias and ReLU: the
// aitrends summary, technical features; it is bound by data movement, the
// activations outweighing the weights 16 to 1: "The Paper Says ARM Support"
// post, "What the model is trying to do".)
//
// k_i8_gemm, persistent, one CTA per SM, 128-token x 128-row output tiles:
//   warp 0     TMA producer: per 128-byte k step one box of xq (128 x 128 B)
//              and one of wq (128 x 128 B), both 128-byte swizzled, into a
//              ring of 4 or 5 stages (k past K and rows past M or N read as
//              zero);
//   warp 1     MMA issuer and TMEM owner: four tcgen05.mma kind::i8 (K = 32
//              each) per stage into one of two 128-column int32 accumulators;
//   warps 2-   epilogue, 8 or 16 warps (2 or 4 per TMEM lane quarter of 32
//              tokens), each taking half or a quarter of the tile's columns:
//              per 32 columns, tcgen05.ld, rescale + bias + ReLU (the tile's
//              bias staged in shared memory), a 128-byte-swizzled 4 KB
//              staging buffer, and a TMA store of the 32 x 32 box (clipped
//              at M and N).  When N is
//              not a multiple of 4 (the output's row pitch is then not a
//              multiple of 16 bytes), the warp stores the staged box with
//              coalesced row writes instead.
// The output is what bounds the layer at the encoder's shapes (4 bytes per
// output against 2 * K int8 operations), so the epilogue keeps several
// stores in flight while the MMAs of the next tile run.  Every wait is
// bounded; on a timeout the block stops, drains its copies and MMAs, frees
// its tensor memory and returns.
#include <cstdio>
#include <cstring>
#include <cuda.h>

#include "tw_device.cuh"
#include "tw_internal.h"
#include "tw_tc.cuh"

namespace tw {
namespace {

constexpr int kBM = 128;                       // tokens per tile (MMA M)
constexpr int kBN = 128;                       // weight rows per tile (MMA N)
constexpr int kBK = 128;                       // bytes of k per stage
constexpr int kABytes = kBM * kBK;             // 16 KB
constexpr int kBBytes = kBN * kBK;             // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiBufs = 1;                    // staging buffer per epilogue warp
constexpr int kBoxBytes = 32 * 32 * 4;         // one 32 x 32 fp32 box
constexpr int kTmemCols = 2 * kBN;

// Launch shapes: EW epilogue warps (8 or 16: EW / 4 per TMEM lane quarter,
// each taking 16 / EW of the quarter's four 32-column boxes of a tile) and
// ST load stages of 128 k bytes.  Measured on B200: with one
// staging buffer per warp, 5 stages beside 8 epilogue warps took the
// 32768 x 512 -> 2048 layer from 87.8 to 68.0 us (3 stages and 3 buffers
// before: a K of 4 stages per tile left the load latency exposed) and left
// 16384 x 256 -> 1024 at 20.6 us; 16 epilogue warps beside 4 stages took
// that one to 18.7 us (K of 2 stages per tile: the epilogue bounds it) but
// the other to 77.0 us.
template <int EW, int ST>
struct I8Shape {
    static_assert(EW % 4 == 0 && 16 % EW == 0, "epilogue warps");
    static constexpr int kEpiWarps = EW, kStages = ST, kBoxesPerWarp = 16 / EW;
    static constexpr int kThreads = (2 + EW) * 32;
    static constexpr int kSmemBytes =
        1024 + ST * kStageBytes + EW * kEpiBufs * kBoxBytes + 1024 + EW * 64 * 4;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};
constexpr uint64_t kDrainNs = 1000000000ull;

struct alignas(64) I8Params {
    CUtensorMap tmap_x;     // xq [M x K] uint8, box 128 x 128, 128-byte swizzle
    CUtensorMap tmap_w;     // wq [N x K] uint8, box 128 x 128, 128-byte swizzle
    CUtensorMap tmap_y;     // y [M x N] fp32, box 32 x 32, 128-byte swizzle (tma_out)
    CUtensorMap tmap_acc;   // acc_out [M x N] int32, same box (tma_out and acc_out)
    const float *amax_x;
    const float *amax_w;
    const float *bias;      // [N] or null
    float *y;
    int32_t *acc_out;       // [M x N] or null
    int64_t M, N, K;
    int64_t tiles_m, tiles;
    int relu;
    int tma_out;            // 1: TMA stores; 0: coalesced row stores
    WaitCtl ctl;
};

// Instruction descriptor: int8 x int8 -> int32, both K-major, M = 128, N = 128.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                              ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ void tile_coords(const I8Params &p, int64_t t, int64_t &mi, int64_t &nj)
{
    // consecutive tiles share a weight tile: the token tiles of one weight
    // tile run side by side across the grid
    nj = t / p.tiles_m;
    mi = t - nj * p.tiles_m;
}

template <int EW, int ST>
__global__ void __launch_bounds__(I8Shape<EW, ST>::kThreads, 1) k_i8_gemm(const __grid_constant__ I8Params p)
{
    constexpr int kEpiWarps = EW, kStages = ST, kBoxesPerWarp = I8Shape<EW, ST>::kBoxesPerWarp;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gen_base = smem_raw + (base - raw);
    const uint32_t stg0 = base + kStages * kStageBytes;
    uint8_t *misc = gen_base + kStages * kStageBytes + kEpiWarps * kEpiBufs * kBoxBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t b_full = bar0, b_empty = bar0 + 8 * kStages;
    const uint32_t b_tfull = bar0 + 16 * kStages, b_tempty = b_tfull + 16;
    const uint32_t b_drain = b_tempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 512);
    int *abort_p = reinterpret_cast<int *>(misc + 520);
    volatile int *abort_flag = abort_p;
    float *bias_s = reinterpret_cast<float *>(misc + 1024);   // [kEpiWarps][64]: per warp

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_tfull + 8 * a, 1);
            mbar_init(b_tempty + 8 * a, kEpiWarps);
        }
        mbar_init(b_drain, 1);
        *abort_p = 0;
        fence_barrier_init();
    }
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t G = gridDim.x;
    const int64_t KT = (p.K + kBK - 1) / kBK;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += G) {
                int64_t mi, nj;
                tile_coords(p, t, mi, nj);
                for (int64_t kt = 0; kt < KT; ++kt, ++it) {
                    const int s = (int)(it % kStages);
                    if (it >= kStages &&
                        !mbar_wait(b_empty + 8 * s, (uint32_t)((it / kStages - 1) & 1), p.ctl,
                                   abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_s = base + s * kStageBytes;
                    mbar_arrive_expect_tx(b_full + 8 * s, (uint32_t)kStageBytes);
                    tma_load_2d(a_s, &p.tmap_x, (int32_t)(kt * kBK), (int32_t)(mi * kBM), b_full + 8 * s);
                    tma_load_2d(a_s + kABytes, &p.tmap_w, (int32_t)(kt * kBK), (int32_t)(nj * kBN),
                                b_full + 8 * s);
                }
            }
            // Drain: the last loads land before the block exits.
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            for (int64_t j = it - kStages; j < it; ++j)
                if (j >= 0)
                    mbar_wait(b_full + 8 * (int)(j % kStages), (uint32_t)((j / kStages) & 1), drain,
                              nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int64_t it = 0, tt = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += G, ++tt) {
                const int ab = (int)(tt & 1);
                if (tt >= 2 &&
                    !mbar_wait(b_tempty + 8 * ab, (uint32_t)((tt / 2 - 1) & 1), p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(ab * kBN);
                for (int64_t kt = 0; kt < KT; ++kt, ++it) {
                    const int s = (int)(it % kStages);
                    if (!mbar_wait(b_full + 8 * s, (uint32_t)((it / kStages) & 1), p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sdesc_k_sw128(base + s * kStageBytes);
                    const uint64_t bd = sdesc_k_sw128(base + s * kStageBytes + kABytes);
#pragma unroll
                    for (int j = 0; j < kBK / 32; ++j)  // +32 bytes of K = +2 in the address field
                        mma_i8(d_tmem, ad + 2 * j, bd + 2 * j, kIdescI8, (kt > 0 || j > 0) ? 1u : 0u);
                    mma_commit(b_empty + 8 * s);
                }
                if (!ok)
                    break;
                mma_commit(b_tfull + 8 * ab);
            }
            // Every MMA issued by this thread completes before TMEM is freed.
            mma_commit(b_drain);
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            mbar_wait(b_drain, 0, drain, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;          // TMEM lanes 32q .. 32q + 31
        const int ew = warp - 2;
        const int half = ew >> 2;              // columns [32 B half, 32 B (half + 1)) of the tile, B = kBoxesPerWarp
        const uint32_t stg = stg0 + (uint32_t)(ew * kEpiBufs * kBoxBytes);
        float *stg_f = reinterpret_cast<float *>(gen_base + (stg - base));
        const float sw = __fdiv_rn(__ldg(p.amax_w), 127.f);
        int64_t tt = 0;
        int nbox = 0;                           // boxes this warp has staged
        // The per-token scale and this half's bias columns of a tile are
        // loaded one tile ahead, so that their L2 round trip overlaps the
        // previous tile's epilogue instead of preceding this one's.
        float amax_n = 0.f, bias_n0 = 0.f, bias_n1 = 0.f;
        auto load_scales = [&](int64_t t) {
            if (t >= p.tiles)
                return;
            int64_t mi, nj;
            tile_coords(p, t, mi, nj);
            const int64_t m = mi * kBM + 32 * quarter + lane;
            const int64_t n = nj * kBN + 32 * kBoxesPerWarp * half + lane;
            amax_n = m < p.M ? __ldg(p.amax_x + m) : 0.f;
            bias_n0 = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.f;
            bias_n1 = (kBoxesPerWarp > 1 && p.bias && n + 32 < p.N) ? __ldg(p.bias + n + 32) : 0.f;
        };
        load_scales(blockIdx.x);
        for (int64_t t = blockIdx.x; t < p.tiles; t += G, ++tt) {
            int64_t mi, nj;
            tile_coords(p, t, mi, nj);
            const int ab = (int)(tt & 1);
            const int64_t m0 = mi * kBM + 32 * quarter;   // first token row of this warp
            const int64_t m = m0 + lane;
            const float sa = m < p.M ? __fdiv_rn(amax_n, 127.f) : 0.f;
            // this half's bias columns into the warp's own shared buffer
            // (the warp's previous tile is done with it)
            float *bias_t = bias_s + 64 * ew;
            bias_t[lane] = bias_n0;
            bias_t[lane + 32] = bias_n1;
            __syncwarp();
            load_scales(t + G);
            if (!mbar_wait(b_tfull + 8 * ab, (uint32_t)((tt / 2) & 1), p.ctl, abort_flag))
                break;
            tc_fence_after();
            for (int hc = 0; hc < kBoxesPerWarp; ++hc) {
                const int cc = kBoxesPerWarp * half + hc;
                const int64_t n0 = nj * kBN + 32 * cc;
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(ab * kBN + 32 * cc), v);
                if (hc == kBoxesPerWarp - 1) {
                    // the accumulator has been read: release it to the MMA warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(b_tempty + 8 * ab);
                }
                if (n0 >= p.N || m0 >= p.M)
                    continue;   // (uniform across the warp)
                const float4 *bias4 = reinterpret_cast<const float4 *>(bias_t + 32 * hc);
                for (int pass = 0; pass < (p.acc_out ? 2 : 1); ++pass) {
                    const int b = nbox % kEpiBufs;
                    const uint32_t box = stg + (uint32_t)(b * kBoxBytes);
                    float *box_f = stg_f + b * (kBoxBytes / 4);
                    if (lane == 0)
                        bulk_wait_group_read<kEpiBufs - 1>();   // this buffer's last store has read it
                    __syncwarp();
                    // row `lane`, 16-byte chunk c at (c ^ (lane & 7)): the 128-byte swizzle
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float4 f;
                        float *fp = reinterpret_cast<float *>(&f);
                        const float4 b4 = bias4[c];   // (one broadcast read)
                        const float *bp = reinterpret_cast<const float *>(&b4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 4 * c + e;
                            const int a = (int)v[j];
                            if (pass == 0) {
                                float yv = __fadd_rn(__fmul_rn(__fmul_rn((float)a, sa), sw), bp[e]);
                                if (p.relu && yv < 0.f)
                                    yv = 0.f;
                                fp[e] = yv;
                            } else {
                                fp[e] = __int_as_float(a);
                            }
                        }
                        *reinterpret_cast<float4 *>(box_f + lane * 32 + ((c ^ (lane & 7)) << 2)) = f;
                    }
                    if (p.tma_out) {
                        fence_proxy_async_smem();   // the box is visible to the TMA engine
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(pass == 0 ? &p.tmap_y : &p.tmap_acc, box, (int32_t)n0,
                                         (int32_t)m0);
                            bulk_commit_group();
                        }
                    } else {
                        __syncwarp();
                        float *dst = pass == 0 ? p.y : reinterpret_cast<float *>(p.acc_out);
                        for (int r = 0; r < 32; ++r) {
                            const int64_t mm = m0 + r, nn = n0 + lane;
                            if (mm < p.M && nn < p.N)
                                dst[mm * p.N + nn] =
                                    box_f[r * 32 + ((((lane >> 2) ^ (r & 7))) << 2) + (lane & 3)];
                        }
                        __syncwarp();
                    }
                    ++nbox;
                }
            }
        }
        if (lane == 0)
            bulk_wait_group_all();   // every store has completed before the block exits
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- weights
// max|W| over the tensor as the bits of a non-negative float (ordered like
// the floats themselves), into *amax_bits (zeroed before the launch).
__global__ void k_absmax(const float4 *__restrict__ W4, int64_t n4, unsigned *amax_bits, uint32_t *err)
{
    float a = 0.f;
    bool finite = true;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = __ldg(W4 + i);
        finite &= isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0)
        atomicMax(amax_bits, __float_as_uint(a));
    if (!finite)
        atomicOr(err, EFLAG_NONFINITE);
}

// wq = clamp(rint(W * (127 / amax)), -128, 127) with one fp32 multiply and
// an IEEE division, half to even; amax == 0 gives wq == 0.
__global__ void k_quant_weights(const float4 *__restrict__ W4, int64_t n4, const float *amax,
                                uint32_t *__restrict__ wq4)
{
    const float a = *amax;
    const bool zero = a == 0.f;
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = __ldg(W4 + i);
        int q[4] = {0, 0, 0, 0};
        if (!zero) {
            q[0] = min(max(__float2int_rn(__fmul_rn(v.x, scale)), -128), 127);
            q[1] = min(max(__float2int_rn(__fmul_rn(v.y, scale)), -128), 127);
            q[2] = min(max(__float2int_rn(__fmul_rn(v.z, scale)), -128), 127);
            q[3] = min(max(__float2int_rn(__fmul_rn(v.w, scale)), -128), 127);
        }
        wq4[i] = (uint32_t)(q[0] & 0xff) | ((uint32_t)(q[1] & 0xff) << 8) |
                 ((uint32_t)(q[2] & 0xff) << 16) | ((uint32_t)(q[3] & 0xff) << 24);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess && f)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// A row-major [rows x cols] matrix of `esize`-byte elements as a 2-D tensor
// map with a (box_c x box_r) box and the 128-byte swizzle.
int encode_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *ptr, int64_t rows,
              int64_t cols, uint32_t box_c, uint32_t box_r)
{
    EncodeTiledFn fn = encoder();
    if (!fn)
        return -1;
    memset(m, 0, sizeof(*m));
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(cols * esize)};
    const cuuint32_t box[2] = {box_c, box_r};
    const cuuint32_t estr[2] = {1, 1};
    return (int)fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr uint64_t kWaitNsI8 = 1000000000ull;

int i8_shape(const char *fn, int64_t M, int64_t N, int64_t K)
{
    char msg[160];
    if (M < 1 || N < 1 || K < 1 || K % 16 || M > (1 << 24) || N > (1 << 24) || K > (1 << 20)) {
        snprintf(msg, sizeof msg, "%s: need M, N >= 1 (<= 2^24) and K a positive multiple of 16 "
                 "(<= 2^20); got M=%lld N=%lld K=%lld", fn, (long long)M, (long long)N,
                 (long long)K);
        return record_error(TW_ERR_SHAPE, msg);
    }
    return TW_OK;
}


template <int EW, int ST>
cudaError_t launch_i8_shape(const I8Params &p, int grid, cudaStream_t stream)
{
    using S = I8Shape<EW, ST>;
    cudaError_t e = cudaFuncSetAttribute(k_i8_gemm<EW, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::kSmemBytes);
    if (e != cudaSuccess)
        return e;
    k_i8_gemm<EW, ST><<<(unsigned)grid, S::kThreads, S::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

int launch_i8(const int8_t *xq, const float *amax_x, int64_t M, int64_t N, int64_t K,
              const int8_t *wq, const float *amax_w, const float *bias, int relu, float *y,
              int32_t *acc_out, cudaStream_t stream)
{
    uint32_t *err = nullptr;
    if (int rc = error_word(&err))
        return rc;
    I8Params p;
    memset(&p, 0, sizeof(p));
    int rc = encode_2d(&p.tmap_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, M, K, kBK, kBM);
    if (!rc)
        rc = encode_2d(&p.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, N, K, kBK, kBN);
    p.tma_out = (N % 4) == 0;
    if (!rc && p.tma_out)
        rc = encode_2d(&p.tmap_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, y, M, N, 32, 32);
    if (!rc && p.tma_out && acc_out)
        rc = encode_2d(&p.tmap_acc, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, acc_out, M, N, 32, 32);
    if (rc) {
        char msg[96];
        snprintf(msg, sizeof msg, "cuTensorMapEncodeTiled failed (%d)", rc);
        return record_error(TW_ERR_CUDA, msg);
    }
    p.amax_x = amax_x;
    p.amax_w = amax_w;
    p.bias = bias;
    p.y = y;
    p.acc_out = acc_out;
    p.M = M;
    p.N = N;
    p.K = K;
    p.tiles_m = (M + kBM - 1) / kBM;
    p.tiles = p.tiles_m * ((N + kBN - 1) / kBN);
    p.relu = relu ? 1 : 0;
    p.ctl.err = err;
    p.ctl.timeout_ns = kWaitNsI8;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return record_error(TW_ERR_CUDA, cudaGetErrorString(e));
    const int64_t grid = p.tiles < sms ? p.tiles : sms;
    // K of at most two stages per tile: the epilogue bounds the layer
    if (K <= 2 * kBK)
        e = launch_i8_shape<16, 4>(p, (int)grid, stream);
    else
        e = launch_i8_shape<8, 5>(p, (int)grid, stream);
    return e == cudaSuccess ? TW_OK : record_error(TW_ERR_CUDA, cudaGetErrorString(e));
}

}  // namespace
}  // namespace tw

extern "C" {

size_t tw_i8_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 1 || K < 1)
        return 0;
    return (size_t)((M * K + 255) / 256 * 256 + (4 * M + 255) / 256 * 256);
}

TW_API int tw_i8_quantize_weights(const float *W, int64_t N, int64_t K, int8_t *wq, float *amax_w,
                                  tw_stream_t stream)
{
    tw::clear_error();
    if (!W || !wq || !amax_w)
        return tw::record_error(TW_ERR_NULL, "tw_i8_quantize_weights: W, wq and amax_w are required");
    if (N < 1 || K < 1 || K % 16 || N > (1 << 24) || K > (1 << 20))
        return tw::record_error(TW_ERR_SHAPE, "tw_i8_quantize_weights: need N >= 1 and K a positive "
                                "multiple of 16");
    if (!tw::aligned16(W) || !tw::aligned16(wq) || !tw::aligned16(amax_w))
        return tw::record_error(TW_ERR_ALIGN, "tw_i8_quantize_weights: pointers must be 16-byte aligned");
    uint32_t *err = nullptr;
    if (int rc = tw::error_word(&err))
        return rc;
    const int64_t n4 = N * K / 4;
    const int64_t blocks64 = (n4 + 255) / 256;
    const unsigned blocks = (unsigned)(blocks64 < 148 * 8 ? blocks64 : 148 * 8);
    cudaError_t e = cudaMemsetAsync(amax_w, 0, sizeof(float), stream);
    if (e == cudaSuccess) {
        tw::k_absmax<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(W), n4,
                                                 reinterpret_cast<unsigned *>(amax_w), err);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        tw::k_quant_weights<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(W), n4,
                                                        amax_w, reinterpret_cast<uint32_t *>(wq));
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? TW_OK : tw::record_error(TW_ERR_CUDA, cudaGetErrorString(e));
}

TW_API int tw_i8_linear_q(const int8_t *xq, const float *amax_x, int64_t M, int64_t N, int64_t K,
                          const int8_t *wq, const float *amax_w, const float *bias, int relu,
                          float *y, int32_t *acc_out, tw_stream_t stream)
{
    tw::clear_error();
    if (!xq || !amax_x || !wq || !amax_w || !y)
        return tw::record_error(TW_ERR_NULL, "tw_i8_linear_q: xq, amax_x, wq, amax_w and y are required");
    if (int rc = tw::i8_shape("tw_i8_linear_q", M, N, K))
        return rc;
    if (!tw::aligned16(xq) || !tw::aligned16(amax_x) || !tw::aligned16(wq) ||
        !tw::aligned16(amax_w) || !tw::aligned16(y) || (bias && !tw::aligned16(bias)) ||
        (acc_out && !tw::aligned16(acc_out)))
        return tw::record_error(TW_ERR_ALIGN, "tw_i8_linear_q: pointers must be 16-byte aligned");
    return tw::launch_i8(xq, amax_x, M, N, K, wq, amax_w, bias, relu, y, acc_out, stream);
}

TW_API int tw_i8_linear(const float *x, int64_t M, int64_t N, int64_t K, const int8_t *wq,
                        const float *amax_w, const float *bias, int relu, float *y,
                        int32_t *acc_out, void *ws, size_t ws_bytes, tw_stream_t stream)
{
    tw::clear_error();
    if (!x || !wq || !amax_w || !y)
        return tw::record_error(TW_ERR_NULL, "tw_i8_linear: x, wq, amax_w and y are required");
    if (int rc = tw::i8_shape("tw_i8_linear", M, N, K))
        return rc;
    if (!ws || ws_bytes < tw_i8_workspace_bytes(M, K))
        return tw::record_error(TW_ERR_BUFSIZE, "tw_i8_linear: workspace smaller than "
                                "tw_i8_workspace_bytes(M, K)");
    if (!tw::aligned16(x) || !tw::aligned16(ws) || !tw::aligned16(wq) || !tw::aligned16(amax_w) ||
        !tw::aligned16(y) || (bias && !tw::aligned16(bias)) || (acc_out && !tw::aligned16(acc_out)))
        return tw::record_error(TW_ERR_ALIGN, "tw_i8_linear: pointers must be 16-byte aligned");
    uint32_t *err = nullptr;
    if (int rc = tw::error_word(&err))
        return rc;
    int8_t *xq = static_cast<int8_t *>(ws);
    float *amax_x = reinterpret_cast<float *>(static_cast<char *>(ws) + (M * K + 255) / 256 * 256);
    cudaError_t e = tw::launch_quantize(x, M, K, xq, amax_x, nullptr, stream);
    if (e != cudaSuccess)
        return tw::record_error(TW_ERR_CUDA, cudaGetErrorString(e));
    return tw::launch_i8(xq, amax_x, M, N, K, wq, amax_w, bias, relu, y, acc_out, stream);
}

}  // extern "C"
