// tw_prefill.cu — ternary GEMM for prefill (M > 32 tokens) on the 5th-
// generation tensor cores (tcgen05, int8, int32 accumulators in TMEM).
//
// D[m, n] = sum_k xq[m, k] * (code[n, k] + 1) runs as tcgen05.mma kind::i8
// (A = int8 activations, K-major, loaded by TMA with 128-byte swizzle;
// B = codes + 1 expanded from the 2-bit layout into int8 in shared memory by
// eight expansion warps), then the epilogue removes the +1 offset with the
// per-token sum(q) and rescales:
//   acc = D - qsum[m],   y = ((float)acc * (amax[m] / 127)) * mean|W|.
// (Per-tensor ternary weights, s = 1/mean|W|: "VibeVoice-ASR-BitNet-ONNX"
// model page, Quantization table.  The prefill length is the audio frame
// count plus the prompt, one frame per 3200 samples of 24 kHz audio: same
// page, "Layout".)
//
// Tile: 128 tokens x 256 weight rows, K in stages of 128 (one swizzle atom),
// four MMAs of K = 32 per stage; five stages of A + code tiles in flight,
// two expanded B tiles (measured on B200: the A + code ring, whose stages
// are held from the TMA issue until their MMAs complete, is the deeper
// need: 398 against 424 us at 256 tokens and 1.40 against 1.47 ms at 1024
// over the 196 projections).  Persistent: one CTA per SM walks the
// output tiles of every projection (all token tiles of a weight tile run
// back to back across the grid, so the weight codes stream from HBM once
// and the activations stay in L2).  Two TMEM accumulators let the epilogue
// of one tile overlap the main loop of the next.
//
// Warps: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2..5 epilogue
// (TMEM lane quarters 2, 3, 0, 1), 6..13 code expansion.  Every wait is
// bounded; on a timeout the block stops, drains its copies and MMAs, frees
// its TMEM and returns.
#include <cstring>
#include <cuda.h>

#include "tw_device.cuh"
#include "tw_internal.h"
#include "tw_tc.cuh"

namespace tw {
namespace {

constexpr int kBM = 128;                 // tokens per tile (MMA M)
constexpr int kBN = 256;                 // weight rows per tile (MMA N)
constexpr int kBK = 128;                 // k per stage
constexpr int kLoadStages = 5;           // A + code tiles in flight
constexpr int kBStages = 2;              // expanded B tiles
constexpr int kABytes = kBM * kBK;       // 16 KB
constexpr int kBBytes = kBN * kBK;       // 32 KB
constexpr int kCodeBytes = kBN / kTileRows * kTileBytes;  // 16 tiles = 8 KB
constexpr int kLoadBytes = kABytes + kCodeBytes;
constexpr int kNumExp = 8;               // expansion warps
constexpr int kThreads = (6 + kNumExp) * 32;
constexpr int kTmemCols = 512;           // two 256-column accumulators
constexpr int kStageRowF = 36;           // epilogue staging row (floats), 32 + 4 pad
constexpr int kStagingBytes = 4 * 32 * kStageRowF * 4;
constexpr int kSmemBytes = 1024 + kLoadStages * kLoadBytes + kBStages * kBBytes + kStagingBytes + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr uint64_t kDrainNs = 1000000000ull;

struct PrefillParams {
    const DescRecord *table;  // null: use `single`
    DescRecord single;
    int count;
    int64_t M;
    int64_t total_ptiles;
    WaitCtl ctl;
};

__device__ __forceinline__ const DescRecord &prec(const PrefillParams &p, int d)
{
    return p.table ? p.table[d] : p.single;
}

// Walks this CTA's output tiles t = blockIdx.x, +G, ... in order, keeping
// the fields of the current projection in registers (no search per tile).
// Inside a projection the token tiles of one weight tile are consecutive:
// local tile = nj * tm + mi.
struct TileIter {
    int64_t t, ptile_end, tm;
    int d;
    int64_t mi, nj, K, N;
    const DescRecord *r;

    __device__ void load(const PrefillParams &p)
    {
        r = &prec(p, d);
        K = r->K;
        N = r->N;
        ptile_end = r->ptile_begin + tm * ((N + kBN - 1) / kBN);
    }
    __device__ void locate(const PrefillParams &p)
    {
        while (t >= ptile_end && d + 1 < p.count) {
            ++d;
            load(p);
        }
        const int64_t local = t - r->ptile_begin;
        mi = local % tm;
        nj = local / tm;
    }
    __device__ void init(const PrefillParams &p, int64_t t0)
    {
        t = t0;
        tm = (p.M + kBM - 1) / kBM;
        d = 0;
        load(p);
        if (t < p.total_ptiles)
            locate(p);
    }
    __device__ bool valid(const PrefillParams &p) const { return t < p.total_ptiles; }
    __device__ void next(const PrefillParams &p, int64_t G)
    {
        t += G;
        if (t < p.total_ptiles)
            locate(p);
    }
};

// Instruction descriptor: int8 x int8 -> int32, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (2u << 4)            // D format: s32
                            | (1u << 7)          // A: signed int8
                            | (1u << 10)         // B: signed int8
                            | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

struct SmemLayout {
    uint32_t base;  // 1024-aligned shared address
    __device__ uint32_t a(int s) const { return base + s * kLoadBytes; }
    __device__ uint32_t codes(int s) const { return base + s * kLoadBytes + kABytes; }
    __device__ uint32_t b(int s) const { return base + kLoadStages * kLoadBytes + s * kBBytes; }
    __device__ uint32_t staging(int w) const
    {
        return base + kLoadStages * kLoadBytes + kBStages * kBBytes + w * (32 * kStageRowF * 4);
    }
};

__global__ void __launch_bounds__(kThreads, 1) k_prefill(const __grid_constant__ PrefillParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gen_base = smem_raw + (base - raw);
    SmemLayout L{base};
    uint8_t *misc = gen_base + kLoadStages * kLoadBytes + kBStages * kBBytes + kStagingBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
    // barriers: ld_full[kLoadStages], ld_empty[kLoadStages], b_full[kBStages],
    // b_empty[kBStages], tmem_full[2], tmem_empty[2], drain
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t b_ldfull = bar0, b_ldempty = bar0 + 8 * kLoadStages;
    const uint32_t b_bfull = bar0 + 16 * kLoadStages, b_bempty = b_bfull + 8 * kBStages;
    const uint32_t b_tfull = b_bempty + 8 * kBStages, b_tempty = b_tfull + 16;
    const uint32_t b_drain = b_tempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 512);
    int *abort_flag_p = reinterpret_cast<int *>(misc + 520);
    volatile int *abort_flag = abort_flag_p;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kLoadStages; ++s) {
            mbar_init(b_ldfull + 8 * s, 1);
            mbar_init(b_ldempty + 8 * s, 1);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(b_bfull + 8 * s, kNumExp * 32);
            mbar_init(b_bempty + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_tfull + 8 * a, 1);
            mbar_init(b_tempty + 8 * a, 4 * 32);
        }
        mbar_init(b_drain, 1);
        *abort_flag_p = 0;
        fence_barrier_init();
    }
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t G = gridDim.x;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int64_t it = 0;
            TileIter ti;
            for (ti.init(p, blockIdx.x); ti.valid(p) && !*abort_flag; ti.next(p, G)) {
                const int64_t KT = ti.K / kBK;
                const int32_t rb0 = (int32_t)(ti.nj * (kBN / kTileRows));
                // the code box is always 16 row blocks (rows past N read as
                // zero and only feed output columns that are not stored)
                const uint32_t bytes = kABytes + kCodeBytes;
                const void *tmap = ti.r->tmap_xq;
                const void *tmap_c = ti.r->tmap_codes;
                const int32_t ycoord = (int32_t)(ti.mi * kBM);
                bool ok = true;
                for (int64_t kt = 0; kt < KT; ++kt, ++it) {
                    const int s = (int)(it % kLoadStages);
                    if (it >= kLoadStages &&
                        !mbar_wait(b_ldempty + 8 * s, (uint32_t)((it / kLoadStages - 1) & 1), p.ctl,
                                   abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(b_ldfull + 8 * s, bytes);
                    tma_load_2d(L.a(s), tmap, (int32_t)(kt * kBK), ycoord, b_ldfull + 8 * s);
                    tma_load_3d(L.codes(s), tmap_c, 0, (int32_t)kt, rb0, b_ldfull + 8 * s);
                }
                if (!ok)
                    break;
            }
            // Drain: the last (up to) kLoadStages loads must land before exit.
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            for (int64_t j = it - kLoadStages; j < it; ++j)
                if (j >= 0)
                    mbar_wait(b_ldfull + 8 * (int)(j % kLoadStages),
                              (uint32_t)((j / kLoadStages) & 1), drain, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int64_t it = 0, tt = 0;
            bool ok = true;
            TileIter ti;
            for (ti.init(p, blockIdx.x); ti.valid(p) && ok; ti.next(p, G), ++tt) {
                const int64_t KT = ti.K / kBK;
                const int ab = (int)(tt & 1);
                if (tt >= 2 && !mbar_wait(b_tempty + 8 * ab, (uint32_t)((tt / 2 - 1) & 1), p.ctl,
                                          abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(ab * kBN);
                for (int64_t kt = 0; kt < KT; ++kt, ++it) {
                    const int ls = (int)(it % kLoadStages), bs = (int)(it % kBStages);
                    if (!mbar_wait(b_ldfull + 8 * ls, (uint32_t)((it / kLoadStages) & 1), p.ctl,
                                   abort_flag) ||
                        !mbar_wait(b_bfull + 8 * bs, (uint32_t)((it / kBStages) & 1), p.ctl,
                                   abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sdesc_k_sw128(L.a(ls));
                    const uint64_t bd = sdesc_k_sw128(L.b(bs));
#pragma unroll
                    for (int j = 0; j < kBK / 32; ++j)  // +32 bytes of K = +2 in the address field
                        mma_i8(d_tmem, ad + 2 * j, bd + 2 * j, kIdesc, (kt > 0 || j > 0) ? 1u : 0u);
                    mma_commit(b_ldempty + 8 * ls);
                    mma_commit(b_bempty + 8 * bs);
                }
                if (!ok)
                    break;
                mma_commit(b_tfull + 8 * ab);
            }
            // All MMAs issued by this thread complete before TMEM is freed.
            mma_commit(b_drain);
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            mbar_wait(b_drain, 0, drain, nullptr);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------ epilogue
        // Each warp owns TMEM lanes 32q..32q+31 (q = warp % 4): 32 token rows
        // of the tile.  Per 32-column chunk: TMEM -> registers (thread = row),
        // rescale, registers -> staging (row-major), then staging -> global
        // with 4 rows x 128 contiguous bytes per store instruction.
        const int quarter = warp & 3;
        const uint32_t stg = L.staging(warp - 2);
        float *stg_f = reinterpret_cast<float *>(gen_base + (stg - base));
        int64_t tt = 0;
        TileIter ti;
        for (ti.init(p, blockIdx.x); ti.valid(p); ti.next(p, G), ++tt) {
            const DescRecord &r = *ti.r;
            const int ab = (int)(tt & 1);
            const int64_t m_base = ti.mi * kBM + quarter * 32;   // first row of this warp
            const int64_t m = m_base + lane;
            const bool row_ok = m < p.M;
            // per-row and per-tensor scales (loaded before the wait)
            const float sa = row_ok ? __fdiv_rn(__ldg(r.amax + m), 127.f) : 0.f;
            const int qs = row_ok ? __ldg(r.qsum + m) : 0;
            const float wscale = __ldg(r.wscale);
            float *const y = r.y;
            int32_t *const acc_out = r.acc_out;
            const int64_t N = ti.N;
            const int64_t n0 = ti.nj * kBN;
            if (!mbar_wait(b_tfull + 8 * ab, (uint32_t)((tt / 2) & 1), p.ctl, abort_flag))
                break;
            tc_fence_after();
            const bool vec = (N & 3) == 0;
            for (int cc = 0; cc < kBN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * kBN + cc * 32), v);
                const int64_t nb = n0 + cc * 32;
                if (nb >= N)
                    continue;  // (uniform across the warp)
                // pass 0: y, pass 1: acc_out
                for (int pass = 0; pass < (acc_out ? 2 : 1); ++pass) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 f;
                        int a0 = (int)v[4 * q + 0] - qs, a1 = (int)v[4 * q + 1] - qs;
                        int a2 = (int)v[4 * q + 2] - qs, a3 = (int)v[4 * q + 3] - qs;
                        if (pass == 0) {
                            f = make_float4(__fmul_rn(__fmul_rn((float)a0, sa), wscale),
                                            __fmul_rn(__fmul_rn((float)a1, sa), wscale),
                                            __fmul_rn(__fmul_rn((float)a2, sa), wscale),
                                            __fmul_rn(__fmul_rn((float)a3, sa), wscale));
                        } else {
                            f = make_float4(__int_as_float(a0), __int_as_float(a1),
                                            __int_as_float(a2), __int_as_float(a3));
                        }
                        *reinterpret_cast<float4 *>(stg_f + lane * kStageRowF + 4 * q) = f;
                    }
                    __syncwarp();
                    float *dst = pass == 0 ? y : reinterpret_cast<float *>(acc_out);
                    if (vec && nb + 32 <= N) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int rr = 4 * i + (lane >> 3), c4 = (lane & 7) * 4;
                            const int64_t mm = m_base + rr;
                            if (mm < p.M) {
                                const float4 f =
                                    *reinterpret_cast<const float4 *>(stg_f + rr * kStageRowF + c4);
                                *reinterpret_cast<float4 *>(dst + mm * N + nb + c4) = f;
                            }
                        }
                    } else {
                        for (int rr = 0; rr < 32; ++rr) {
                            const int64_t mm = m_base + rr;
                            if (mm < p.M && nb + lane < N)
                                dst[mm * N + nb + lane] = stg_f[rr * kStageRowF + lane];
                        }
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            mbar_arrive(b_tempty + 8 * ab);
        }
    } else {
        // ------------------------------------------------------ expansion
        const int e = threadIdx.x - 6 * 32;           // 0..255
        int64_t it = 0;
        bool ok = true;
        TileIter ti;
        for (ti.init(p, blockIdx.x); ti.valid(p) && ok; ti.next(p, G)) {
            const int64_t KT = ti.K / kBK;
            for (int64_t kt = 0; kt < KT; ++kt, ++it) {
                const int ls = (int)(it % kLoadStages), bs = (int)(it % kBStages);
                if (!mbar_wait(b_ldfull + 8 * ls, (uint32_t)((it / kLoadStages) & 1), p.ctl,
                               abort_flag) ||
                    (it >= kBStages &&
                     !mbar_wait(b_bempty + 8 * bs, (uint32_t)((it / kBStages - 1) & 1), p.ctl,
                                abort_flag))) {
                    ok = false;
                    break;
                }
                // Two 16-byte lane slots per thread: slot q = e + 256*h is lane
                // l = q % 32 of code tile q / 32 (rows 16*(q/32) .. +15).
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int q = e + 256 * h;
                    const int tile = q >> 5, l = q & 31;
                    const int g = l >> 2, tq = l & 3;
                    const uint4 w = lds128(L.codes(ls) + tile * kTileBytes + l * 16);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = (jj + 2 * (g & 1)) & 3;   // staggered: no bank conflicts
                        const uint32_t wd = j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w;
                        const int row = tile * kTileRows + g + 8 * (j & 1);
                        const int chunk = 4 * (j >> 1) + tq;      // 16-byte chunk of the 128 B row
                        const uint32_t dst = L.b(bs) + row * 128 + ((chunk ^ (row & 7)) << 4);
                        const uint32_t m3 = 0x03030303u;
                        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst),
                                     "r"(wd & m3), "r"((wd >> 2) & m3), "r"((wd >> 4) & m3),
                                     "r"((wd >> 6) & m3)
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();  // make the B tile visible to the tensor cores
                mbar_arrive(b_bfull + 8 * bs);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int encode_xq_tmap(const int8_t *xq, int64_t M, int64_t K, int box_m, void *out128)
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !f)
            return -1;
        fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    CUtensorMap m;
    memset(&m, 0, sizeof(m));
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {kBK, (cuuint32_t)box_m};   // 128 k bytes x box_m tokens
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(xq), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return (int)r;
    static_assert(sizeof(CUtensorMap) == 128, "tensor map size");
    memcpy(out128, &m, sizeof(m));
    return 0;
}

int encode_codes_tmap(const uint8_t *packed, int64_t N, int64_t K, int box_rb, int box_kt,
                      void *out128)
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !f)
            return -1;
        fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    CUtensorMap m;
    memset(&m, 0, sizeof(m));
    const int64_t KT = K / kTileK, nrb = (N + kTileRows - 1) / kTileRows;
    const cuuint64_t dims[3] = {(cuuint64_t)(kTileBytes / 4), (cuuint64_t)KT, (cuuint64_t)nrb};
    const cuuint64_t strides[2] = {(cuuint64_t)kTileBytes, (cuuint64_t)(KT * kTileBytes)};
    const cuuint32_t box[3] = {kTileBytes / 4, (cuuint32_t)box_kt, (cuuint32_t)box_rb};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(packed), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return (int)r;
    memcpy(out128, &m, sizeof(m));
    return 0;
}

int64_t prefill_tiles(int64_t M, int64_t N)
{
    return ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
}

cudaError_t launch_prefill(const PrefillLaunch &L, uint32_t *err, uint64_t timeout_ns,
                           cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    if (L.single)
        p.single = *L.single;
    p.count = L.count;
    p.M = L.M;
    p.total_ptiles = L.total_ptiles;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    const int smem = kSmemBytes;
    e = cudaFuncSetAttribute(k_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    const int64_t grid = L.total_ptiles < sms ? L.total_ptiles : sms;
    k_prefill<<<(unsigned)(grid < 1 ? 1 : grid), kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tw
