// tw_decode.cu — activation quantisation + ternary GEMV for decode (M <= 32
// tokens), as two launches over any number of projections.
//
// What it computes, per projection: q = absmax int8 quantisation of each
// token row of x, acc = q * codes^T in exact integer arithmetic, and
// y = ((float)acc * (amax/127)) * mean|W|.  (Per-tensor ternary weights with
// s = 1/mean|W|: "VibeVoice-ASR-BitNet-ONNX" model page, Quantization table;
// the weights of all 196 projections are read once per token, which is what
// bounds decode: "The Paper Says ARM Support" post, "What the model is
// trying to do".)
//
// Launch 1 (k_quant_rows): 8, 4, 2 or 1 warps per (projection, token) row,
// by the number of rows, quantise the row, held in registers (one HBM round
// trip), into int8 scratch together with amax/127 and sum(q); with many rows
// the large-K rows get a launch of their own at 8 warps per row.  It lets
// launch 2 start at once (programmatic dependent launch), so the weight
// stream below overlaps it.
//
// Launch 2 (k_decode), one CTA per SM:
//   * The grid splits the concatenated 16-row blocks of all projections into
//     shares of equal estimated cost (16 per 128-column tile + a fixed part
//     per row block); each CTA streams its share once.
//   * NC consumer warps (19 for up to 8 tokens, 15 for 9 to 16, 7 above, or
//     fewer as shared memory allows) each own every NC-th row block of the
//     share and keep a private ring of 2 to 3.5 KB slots (by the token
//     count) that they fill with 1-D bulk copies (the TMA engine) ahead of
//     the arithmetic; each tile's lane slot is read from shared memory just
//     before its MMAs (few registers, so more warps fit) and the slot is
//     refilled once the chunk is done.
//   * The last warp (activation warp) waits for launch 1, then bulk-copies each
//     projection's int8 rows, amax/127 and sum(q) into a byte ring in shared
//     memory (entries sized per projection, up to 8 in flight) ahead of the
//     consumers.
//   * Codes are decoded in registers with one AND per register:
//     word & (0x03030303 << 2s) holds four codes + 1 of consecutive k,
//     scaled by 4^s, as unsigned bytes; they feed m16n8k32 u8 x s8 MMAs
//     (weights are the 16-row side, tokens the 8-column side), one
//     accumulator per s.  At the end acc = sum_s (acc_s >> 2s) - sum(q),
//     exact: sum (c+1) q - sum q = sum c q.
//   * Every wait is bounded; a timeout sets the device error word, stops the
//     block and drains the copies still in flight before the block exits.
#include <cstring>

#include "tw_device.cuh"
#include "tw_gemv.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

// Tiles per ring chunk of the register kernel.  Measured on B200 with the
// full-chunk fast path: 7 tiles (3.5 KB; a K = 8960 row block is exactly 10
// chunks) for groups of up to 4 tokens; 6 tiles (3 KB) for 5 to 8 and 17 to
// 32 tokens, whose activation rows need the shared memory; 4 tiles (2 KB)
// for 9 to 16, so that 15 consumer warps fit beside 16 rows of K = 8960 (11
// with 3 KB chunks, 7 with 3.5 KB).  A partial chunk runs as 4 + 2 + 1
// tiles, so a chunk holds at most 8.
constexpr int chunk_tiles(int mg) { return mg <= 4 ? 7 : mg > 8 && mg <= 16 ? 4 : 6; }
constexpr int kXE = 8;                      // activation ring entries
constexpr int kSmemLimit = 227 * 1024;
constexpr int kPC = 32;                     // projections cached in shared memory per block
constexpr int kMiscBytes = 2048 + 256 * kXE + 64 * kPC;  // token info, barriers, plan,
                                                          // entry offsets, projection cache
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr int kQThreads = 256;
constexpr int kQRegs = 9;                   // float4 per thread kept in registers

struct DecodeParams {
    const DescRecord *table;  // null: use `single`
    DescRecord single;
    int count;
    int M;
    int m0, mg;               // token group [m0, m0 + mg)
    int xcap;                 // bytes of the activation ring (multiple of 128)
    int xs;                   // max_K + 64: bytes of the zero row
    int slots;                // ring slots per consumer warp
    int64_t total_rb, total_cost;
    const uint8_t *ws;        // quantised activations (launch 1 output)
    int64_t ws_sa_off;        // offset of the per-projection amax/127, sum(q)
    WaitCtl ctl;
};

struct QuantParams {
    const DescRecord *table;
    DescRecord single;
    int count, M;             // projections of this launch, tokens
    int ntok;                 // 0: plain int8 rows; 8/16/32: tensor-core token blocks
    int wpr;                  // warps per row (set by launch_quant_rows)
    const UnitOrder *order;   // null: projection i is record i; else order[i0 + i].d
    int i0;
    int wait_prev;            // wait for the preceding launch before finishing
    int own;                  // 1: q, amax and sum(q) go to each record's own xq, amax
                              // and qsum (sweeps of more than 32 tokens given fp32 x);
                              // records without x are skipped
    uint8_t *ws;
    int64_t ws_sa_off;
};

struct Plan {
    int64_t rb_lo, rb_hi;
    int d_lo, d_hi;
    int abort_flag;
};

template <class P>
__device__ __forceinline__ const DescRecord &rec(const P &p, int d)
{
    return p.table ? p.table[d] : p.single;
}

__device__ __forceinline__ int64_t rb_count(const DescRecord &r) { return (r.N + 15) >> 4; }

__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ----------------------------------------------------------------- launch 1
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

__device__ __forceinline__ float amax4(float4 v)
{
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// Offset, in the tensor-core token blocks of one projection, of the four
// bytes q[4 idx .. 4 idx + 3] of token m: k tile kt = idx / 32 is a block of
// ntok rows x 128 bytes; logical k group G = idx mod 32 = 16h + 4t + s goes
// to column c = 8s + 2t + h (4 bytes each) of row m, whose 16-byte chunks
// are swizzled by m mod 8.
__device__ __forceinline__ int64_t tc_block_offset(int64_t idx, int m, int ntok)
{
    const int G = (int)(idx & 31);
    const int h = G >> 4, t = (G >> 2) & 3, s = G & 3;
    const int c = 8 * s + 2 * t + h;
    return (idx >> 5) * (int64_t)ntok * 128 + m * 128 + ((((c >> 2) ^ (m & 7)) << 4) | ((c & 3) << 2));
}

// Quantise token row m of projection d.  amax = max|x|, scale = 127/amax
// (IEEE fp32), q = clamp(rint(x*scale), -128, 127).  A row is handled by
// p.wpr warps (1, 2, 4 or 8; more when there are few rows, so that the
// launch fills the GPU in one wave of short rows); a block of 8 warps holds
// 8 / wpr rows.  Each row is held in registers when it fits, else read twice.
// (3 blocks of 8 warps per SM: 80 registers, 9 float4 per thread.  Measured
// on B200 against 2 blocks at 12 float4: the sweep step of 4 / 8 / 16 / 32
// tokens 78.4 / 82.9 / 119.6 / 140.4 -> 76.5 / 81.2 / 117.7 / 135.7 us.)
__global__ void __launch_bounds__(kQThreads, 3) k_quant_rows(const __grid_constant__ QuantParams p)
{
    pdl_launch_dependents();
    __shared__ float red_f[kQThreads / 32];
    __shared__ int red_i[kQThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wpr = p.wpr, rloc = warp / wpr, wr = warp % wpr;
    const int64_t row_id = (int64_t)blockIdx.x * (kQThreads / 32 / wpr) + rloc;
    const bool in_range = row_id < (int64_t)p.count * p.M;
    const int pi = in_range ? (int)(row_id / p.M) : 0, m = in_range ? (int)(row_id % p.M) : 0;
    const int d = p.order ? p.order[p.i0 + pi].d : pi;
    const DescRecord &r = rec(p, d);
    const bool live = in_range && (!p.own || r.x != nullptr);
    const int64_t K4 = live ? r.K / 4 : 0;
    const float4 *row = reinterpret_cast<const float4 *>(r.x + (int64_t)m * r.K);
    uint32_t *qrow = p.own ? reinterpret_cast<uint32_t *>(const_cast<int8_t *>(r.xq) + (int64_t)m * r.K)
                           : reinterpret_cast<uint32_t *>(p.ws + r.ws_xq_off + (int64_t)m * r.K);
    const int T = 32 * wpr, ti = 32 * wr + lane;   // threads of the row, index within it
    const bool in_regs = K4 <= (int64_t)kQRegs * T;

    float4 v[kQRegs];
    float a = 0.f;
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kQRegs; ++i) {
            const int64_t idx = ti + (int64_t)i * T;
            v[i] = idx < K4 ? __ldg(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kQRegs; ++i)
            a = fmaxf(a, amax4(v[i]));
    } else {
        // batches of kQRegs independent loads per thread
        for (int64_t b0 = ti; b0 < K4; b0 += (int64_t)kQRegs * T) {
#pragma unroll
            for (int i = 0; i < kQRegs; ++i) {
                const int64_t idx = b0 + (int64_t)i * T;
                v[i] = idx < K4 ? __ldg(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < kQRegs; ++i)
                a = fmaxf(a, amax4(v[i]));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (wpr > 1) {  // (uniform over the block)
        if (lane == 0)
            red_f[warp] = a;
        __syncthreads();
        a = red_f[rloc * wpr];
        for (int w = 1; w < wpr; ++w)
            a = fmaxf(a, red_f[rloc * wpr + w]);
    }

    const bool zero = (a == 0.f);
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    int sum = 0;
    // Token-block stores: every float4 index of this thread is lane mod 32,
    // so its column and swizzle are fixed; only the k tile (idx / 32) moves.
    uint8_t *const tc_lane = p.ws + r.ws_xq_off + (p.ntok ? tc_block_offset(lane, m, p.ntok) : 0);
    const int64_t tc_tile = (int64_t)p.ntok * 128;
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kQRegs; ++i) {
            const int64_t idx = ti + (int64_t)i * T;
            if (idx < K4) {
                const uint32_t u = quant4(v[i], scale, zero, sum);
                if (p.ntok)
                    *reinterpret_cast<uint32_t *>(tc_lane + (idx >> 5) * tc_tile) = u;
                else
                    qrow[idx] = u;
            }
        }
    } else {
        for (int64_t b0 = ti; b0 < K4; b0 += (int64_t)kQRegs * T) {
#pragma unroll
            for (int i = 0; i < kQRegs; ++i) {
                const int64_t idx = b0 + (int64_t)i * T;
                v[i] = idx < K4 ? __ldg(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < kQRegs; ++i) {
                const int64_t idx = b0 + (int64_t)i * T;
                if (idx < K4) {
                    const uint32_t u = quant4(v[i], scale, zero, sum);
                    if (p.ntok)
                        *reinterpret_cast<uint32_t *>(tc_lane + (idx >> 5) * tc_tile) = u;
                    else
                        qrow[idx] = u;
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (wpr > 1) {
        if (lane == 0)
            red_i[warp] = sum;
        __syncthreads();
        sum = 0;
        for (int w = 0; w < wpr; ++w)
            sum += red_i[rloc * wpr + w];
    }
    if (live && ti == 0) {
        if (p.own) {
            const_cast<float *>(r.amax)[m] = a;
            const_cast<int32_t *>(r.qsum)[m] = sum;
        } else {
            uint8_t *info = p.ws + p.ws_sa_off + 256 * (int64_t)d;
            reinterpret_cast<float *>(info)[m] = __fdiv_rn(a, 127.f);
            reinterpret_cast<int *>(info + 128)[m] = sum;
        }
    }
    // This launch overlaps the preceding one (programmatic dependent launch);
    // it completes only after that one has, so that waiting for this launch
    // covers both.
    if (p.wait_prev)
        pdl_wait();
}

// Warps per row for `rows` rows: enough warps in flight to fill the GPU
// (about 24 resident per SM at this kernel's register use) in one wave.
int quant_warps_per_row(int64_t rows, int sms)
{
    const int64_t target = (int64_t)sms * 24;
    int w = 8;
    while (w > 1 && rows * w > target)
        w >>= 1;
    return w;
}

int sm_count()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

cudaError_t launch_quant_once(const QuantParams &q, bool pdl, cudaStream_t stream)
{
    const int64_t rows = (int64_t)q.count * q.M;
    const int64_t per_block = kQThreads / 32 / q.wpr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows + per_block - 1) / per_block));
    cfg.blockDim = dim3(kQThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_quant_rows, q);
}

// Launches of the quantisation pass: one, or -- when there are so many rows
// that a row would get at most 2 warps, and the large-K rows then need two
// passes over x -- two: the projections of the order with K > kQuantSmallK
// (entries [0, n_big)) at 8 warps per row, so that each row is read once
// into registers, and the rest with as many warps per row as fill the GPU.
// (Measured on B200: the second launch pays off from 8 tokens of the
// 196-projection sweep on, not at 4.)
int quant_launches_impl(int64_t count, int64_t M, int n_big)
{
    const int w = quant_warps_per_row(count * M, sm_count());
    return (w <= 2 && n_big > 0 && n_big < count) ? 2 : 1;
}

cudaError_t launch_quant_rows(QuantParams &q, int n_big, cudaStream_t stream)
{
    const int sms = sm_count();
    if (!q.order || quant_launches_impl(q.count, q.M, n_big) == 1) {
        q.wpr = quant_warps_per_row((int64_t)q.count * q.M, sms);
        q.order = nullptr;   // one launch: the projections in record order
        q.i0 = 0;
        q.wait_prev = 0;
        return launch_quant_once(q, false, stream);
    }
    QuantParams a = q, b = q;
    a.i0 = 0;
    a.count = n_big;
    a.wpr = 8;
    a.wait_prev = 0;
    b.i0 = n_big;
    b.count = q.count - n_big;
    b.wpr = quant_warps_per_row((int64_t)b.count * q.M, sms);
    b.wait_prev = 1;
    cudaError_t e = launch_quant_once(a, false, stream);
    if (e == cudaSuccess)
        e = launch_quant_once(b, true, stream);
    return e;
}

// ----------------------------------------------------------------- launch 2
// Cost of one 16-row block (the host's rb_cost): 16 units per 128-column
// tile plus a fixed part for its epilogue and loop set-up.
__device__ __forceinline__ int64_t rb_cost_dev(int64_t K) { return rb_cost(K); }

// CTA i of G owns the row blocks from the first one whose cost range
// starts at or after floor(total_cost * i / G) up to the next CTA's first.
// Given t = floor(total_cost * i / G) and the projection r whose cost range
// holds t, that first block is:
__device__ __forceinline__ int64_t share_start_in(const DescRecord &r, int64_t t)
{
    const int64_t c = rb_cost_dev(r.K);
    const int64_t rl = (t - r.cost_begin + c - 1) / c;
    return min(r.rb_begin + rl, r.rb_begin + rb_count(r));
}

// The fields of one projection that the decode block needs, copied once
// into shared memory (the first kPC projections of the block's share), so
// that moving to the next projection reads no global memory.
struct ProjC {
    const uint8_t *packed;
    float *y;
    int32_t *acc_out;
    int64_t N;
    int64_t ws_xq_off;
    int rb_begin, rb_end, KT, K;
    float wscale;
    int pad;
};
static_assert(sizeof(ProjC) == 64, "projection cache entry");

__device__ __forceinline__ ProjC load_proj(const DecodeParams &p, int d)
{
    const DescRecord &r = rec(p, d);
    return ProjC{r.packed, r.y, r.acc_out, r.N, r.ws_xq_off, (int)r.rb_begin,
                 (int)(r.rb_begin + rb_count(r)), (int)(r.K / kTileK), (int)r.K, __ldg(r.wscale), 0};
}

// Projection d of a block whose share starts at projection d0: from the
// cache when it is there.
__device__ __forceinline__ ProjC get_proj(const DecodeParams &p, const ProjC *pc, int d0, int npc,
                                          int d)
{
    return d - d0 < npc ? pc[d - d0] : load_proj(p, d);
}

// Walks the chunks of one consumer warp: every NC-th row block of the CTA
// share, each cut into ceil(KT / CT) chunks.  The fields of the current
// projection are cached here so that issuing a chunk reads no global memory.
template <int NC, int CT>
struct ChunkIter {
    const uint8_t *packed;
    int rb, rb_begin, rb_end, rb_hi;   // row-block indices (< 2^31)
    int d, kc, nch, KT;
    bool valid;
    const ProjC *pc;                   // projection cache of the block
    int d0, npc;

    __device__ void load_desc(const DecodeParams &p)
    {
        const ProjC c = get_proj(p, pc, d0, npc, d);
        packed = c.packed;
        rb_begin = c.rb_begin;
        rb_end = c.rb_end;
        KT = c.KT;
        nch = (KT + CT - 1) / CT;
    }
    __device__ void seek(const DecodeParams &p)
    {
        while (rb >= rb_end) {
            ++d;
            load_desc(p);
        }
    }
    __device__ void init(const DecodeParams &p, const Plan &pl, int w, const ProjC *cache,
                         int ncache)
    {
        pc = cache;
        d0 = pl.d_lo;
        npc = ncache;
        rb = (int)pl.rb_lo + w;
        rb_hi = (int)pl.rb_hi;
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
        rb += NC;
        valid = rb < rb_hi;
        if (valid)
            seek(p);
    }
    // Bulk-copy this chunk's tiles into dst, completing on bar.
    __device__ __forceinline__ void issue(uint32_t dst, uint32_t bar) const
    {
        const int kt0 = kc * CT;
        const int n = min(CT, KT - kt0);
        const uint8_t *src =
            packed + ((int64_t)(rb - rb_begin) * KT + kt0) * (int64_t)kTileBytes;
        mbar_arrive_expect_tx(bar, (uint32_t)(n * kTileBytes));
        bulk_g2s(dst, src, (uint32_t)(n * kTileBytes), bar);
    }
};

template <int NT, int NC, int CT>
__global__ void __launch_bounds__((NC + 1) * 32, 1) k_decode(const __grid_constant__ DecodeParams p)
{
    constexpr int kChunk = CT * kTileBytes;  // a multiple of 128
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int kThr = (NC + 1) * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Layout: rings | zero row (at 64 mod 128) | activation ring (xcap bytes,
    // 0 mod 128) | token info | barriers | plan | entry offsets.
    // The activation ring holds one entry per projection in flight: its mg
    // int8 rows at stride K + 64 (rows 64 bytes apart mod 128, so the
    // 16-byte token loads of a warp hit distinct banks), starting at 0 mod
    // 128; entries are allocated in order and freed in order.
    const int ring_bytes = NC * p.slots * kChunk;
    uint8_t *ring = smem;
    uint8_t *zero_row = smem + ring_bytes + 64;
    uint8_t *xbase = smem + ring_bytes + 64 + p.xs;  // = ring + K + 128: 0 mod 128
    uint8_t *misc = xbase + p.xcap + 128;
    misc += (128 - (smem_u32(misc) & 127)) & 127;
    uint8_t *info = misc;                                    // [kXE][256]: sa[32], qs[32]
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc + 256 * kXE);
    // bars: ring_full[NC*slots], x_full[kXE], x_empty[kXE]
    Plan *plan = reinterpret_cast<Plan *>(misc + 256 * kXE + 8 * (NC * p.slots + 2 * kXE));
    volatile int *xoff = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(plan) + 64);
    ProjC *pcache = reinterpret_cast<ProjC *>(reinterpret_cast<uint8_t *>(plan) + 128);
    // the activation ring's entry starts (in shared memory: a local array
    // indexed by entry lands in local memory, which the shared-memory
    // carve-out leaves no L1 for)
    int64_t *xstart = reinterpret_cast<int64_t *>(pcache + kPC);
    const uint32_t bar_ring = smem_u32(bars);
    const uint32_t bar_xfull = bar_ring + 8 * NC * p.slots;
    const uint32_t bar_xempty = bar_xfull + 8 * kXE;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NC * p.slots; ++i)
            mbar_init(bar_ring + 8 * i, 1);
        for (int b = 0; b < kXE; ++b) {
            mbar_init(bar_xfull + 8 * b, 1);
            mbar_init(bar_xempty + 8 * b, NC * 32);
        }
        fence_barrier_init();
        plan->abort_flag = 0;
        if (blockIdx.x == 0) {
            plan->rb_lo = 0;
            plan->d_lo = 0;
        }
        if (blockIdx.x + 1 >= gridDim.x) {
            plan->rb_hi = p.total_rb;
            plan->d_hi = p.count - 1;
        }
    }
    // The share's bounds: every thread tests the projections it holds, so
    // the search costs one round of table loads, not a chain of them (one
    // thread's binary searches, about 36 dependent loads, delayed the first
    // code copies: 72.5 -> 68.3 us per one-token sweep of 196 projections,
    // measured on B200).
    {
        const int G = gridDim.x, c = blockIdx.x;
        const int64_t t_lo = p.total_cost * c / G, t_hi = p.total_cost * (c + 1) / G;
        for (int d = threadIdx.x; d < p.count; d += kThr) {
            const DescRecord &r = rec(p, d);
            const int64_t cb = r.cost_begin;
            const int64_t cn = d + 1 < p.count ? rec(p, d + 1).cost_begin : INT64_MAX;
            // the projections of the share's first and last row blocks: the
            // block starting at t can be the first one after r
            if (c > 0 && cb <= t_lo && t_lo < cn) {
                const int64_t b = share_start_in(r, t_lo);
                plan->rb_lo = b;
                plan->d_lo = b < r.rb_begin + rb_count(r) ? d : d + 1;
            }
            if (c + 1 < G && cb <= t_hi && t_hi < cn) {
                const int64_t b = share_start_in(r, t_hi);
                plan->rb_hi = b;
                plan->d_hi = b > r.rb_begin ? d : d - 1;
            }
        }
    }
    for (int i = threadIdx.x; i < p.xs / 16; i += kThr)
        reinterpret_cast<uint4 *>(zero_row)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    Plan pl = *plan;
    if (pl.rb_lo >= pl.rb_hi) {  // an empty share
        pl.d_lo = 0;
        pl.d_hi = -1;
    }
    volatile int *abort_flag = &plan->abort_flag;
    const int npc = pl.d_hi - pl.d_lo + 1 < kPC ? pl.d_hi - pl.d_lo + 1 : kPC;
    for (int i = threadIdx.x; i < npc; i += kThr)
        pcache[i] = load_proj(p, pl.d_lo + i);
    __syncthreads();

    if (warp == NC) {
        // ------------------------------------------------ activation warp
        if (lane == 0) {
            pdl_wait();  // launch 1 has finished writing the int8 rows
            // Positions are counted monotonically; entry seg lives at
            // start[seg % kXE] mod xcap.  `tail` is the oldest entry not yet
            // known to be free.
            int64_t head = 0;
            int64_t *start = xstart;
            int tail = 0, nissued = 0;
            bool ok = true;
            for (int d = pl.d_lo; d <= pl.d_hi && ok; ++d) {
                const int seg = d - pl.d_lo, e = seg % kXE;
                const ProjC r = get_proj(p, pcache, pl.d_lo, npc, d);
                const int64_t rs = r.K + 64;
                const int64_t size = (p.mg * rs + 127) / 128 * 128;
                int64_t pos = head;
                if (pos % p.xcap + size > p.xcap)  // an entry never wraps
                    pos = (pos / p.xcap + 1) * p.xcap;
                // free entries (in order) until the slot and the bytes are available
                while (tail < seg && (seg - tail >= kXE || pos + size - start[tail % kXE] > p.xcap)) {
                    if (!mbar_wait(bar_xempty + 8 * (tail % kXE), (tail / kXE) & 1, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++tail;
                }
                if (!ok)
                    break;
                start[e] = pos;
                head = pos + size;
                const int off = (int)(pos % p.xcap);
                xoff[e] = off;
                const uint32_t bx = bar_xfull + 8 * e;
                const uint32_t dst = smem_u32(xbase + off);
                mbar_arrive_expect_tx(bx, (uint32_t)(p.mg * r.K + 256));
                for (int tok = 0; tok < p.mg; ++tok)
                    bulk_g2s(dst + tok * (uint32_t)rs, p.ws + r.ws_xq_off + (int64_t)(p.m0 + tok) * r.K,
                             (uint32_t)r.K, bx);
                bulk_g2s(smem_u32(info + 256 * e), p.ws + p.ws_sa_off + 256 * (int64_t)d, 256, bx);
                ++nissued;
            }
            // Drain: the activation copies of the last entries issued land
            // before exit.
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            for (int seg = nissued - kXE; seg < nissued; ++seg)
                if (seg >= 0)
                    mbar_wait(bar_xfull + 8 * (seg % kXE), (seg / kXE) & 1, drain, nullptr);
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int g = lane >> 2, t = lane & 3;
    const int S = p.slots;
    const uint32_t ring_w = smem_u32(ring) + warp * S * kChunk + lane * 16;  // this lane's slot
    const uint32_t ring_w0 = smem_u32(ring) + warp * S * kChunk;
    const uint32_t bar_w = bar_ring + 8 * warp * S;
    const uint32_t zero_s = smem_u32(zero_row);

    ChunkIter<NC, CT> cons, prod;
    cons.init(p, pl, warp, pcache, npc);
    prod = cons;
    int issued = 0, consumed = 0;
    for (int s = 0; s < S && prod.valid; ++s) {
        if (lane == 0)
            prod.issue(ring_w0 + s * kChunk, bar_w + 8 * s);
        prod.next(p);
        ++issued;
    }
    int cslot = 0;
    uint32_t cphase = 0;

    bool ok = true;
    for (int d = pl.d_lo; d <= pl.d_hi && ok; ++d) {
        const int seg = d - pl.d_lo, b = seg % kXE;
        if (!mbar_wait(bar_xfull + 8 * b, (seg / kXE) & 1, p.ctl, abort_flag)) {
            ok = false;
            break;
        }
        // this projection's fields, read once
        const ProjC r = get_proj(p, pcache, pl.d_lo, npc, d);
        const float wscale = r.wscale;
        const int64_t N = r.N, rbeg = r.rb_begin;
        float *const y = r.y;
        int32_t *const acc_out = r.acc_out;
        const float *sa = reinterpret_cast<const float *>(info + 256 * b);
        const int *qs = reinterpret_cast<const int *>(info + 256 * b + 128);
        uint32_t xrow[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tok = 8 * nt + g;
            xrow[nt] = (tok < p.mg ? smem_u32(xbase + xoff[b]) + tok * (uint32_t)(r.K + 64) : zero_s) +
                       16 * t;
        }

        while (cons.valid && cons.d == d) {
            int acc[NT][4][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int s = 0; s < 4; ++s)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        acc[nt][s][i] = 0;
            const int64_t rb = cons.rb;
            const int nch = cons.nch, KT = cons.KT;  // cons moves on after the last chunk
            for (int kc = 0; kc < nch; ++kc) {
                if (!mbar_wait(bar_w + 8 * cslot, cphase, p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                chunk_mma<NT, CT>(acc, ring_w + cslot * kChunk, xrow,
                                  (uint32_t)(kc * CT * kTileK), min(CT, KT - kc * CT));
                __syncwarp();
                if (prod.valid) {
                    if (lane == 0) {
                        fence_proxy_async_smem();
                        prod.issue(ring_w0 + cslot * kChunk, bar_w + 8 * cslot);
                    }
                    prod.next(p);
                    ++issued;
                }
                ++consumed;
                if (++cslot == S) {
                    cslot = 0;
                    cphase ^= 1u;
                }
                cons.next(p);
            }
            if (!ok)
                break;
            // epilogue of row block rb: rows 16*rl + g (+8), tokens 8nt + 2t (+1)
            const int64_t rl = rb - rbeg;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = 8 * nt + 2 * t + (i & 1);
                    const int64_t row = rl * kTileRows + g + 8 * (i >> 1);
                    if (tok < p.mg && row < N) {
                        const int m = p.m0 + tok;  // sa/qs hold all M tokens
                        const int v = acc[nt][0][i] + (acc[nt][1][i] >> 2) +
                                      (acc[nt][2][i] >> 4) + (acc[nt][3][i] >> 6) - qs[m];
                        const int64_t o = (int64_t)m * N + row;
                        y[o] = __fmul_rn(__fmul_rn((float)v, sa[m]), wscale);
                        if (acc_out)
                            acc_out[o] = v;
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
            mbar_wait(bar_w + 8 * (i % S), (i / S) & 1, drain, nullptr);
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

// Consumer warps per block: more warps hide more latency (measured on B200:
// 19 beat 15 by 6 % at one token; 23 spill at the 80 registers they leave;
// for two token tiles 15 beat 11 by 2-5 % at 9 to 16 tokens, in 128
// registers), fewer leave registers for the wider accumulators of larger
// token groups and shared memory for their activation rows.  The block is a multiple of 4
// warps so that each SM sub-partition's register file holds the same number
// of warps.
int max_consumers(int nt) { return nt == 1 ? 19 : nt == 2 ? 15 : 7; }

template <int NT, int NC, int CT>
cudaError_t launch_nt(const DecodeParams &p, int grid, int smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(k_decode<NT, NC, CT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    // Programmatic dependent launch: may start while k_quant_rows runs.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((NC + 1) * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode<NT, NC, CT>, p);
}

// Bytes of dynamic shared memory of k_decode for this plan.
int64_t smem_bytes(int nc, int slots, int ct, int xcap, int64_t max_K)
{
    const int64_t xs = max_K + 64;
    return 1024 + (int64_t)nc * slots * ct * kTileBytes + xs + 128 + xcap + 256 + kMiscBytes;
}

struct DecodePlan {
    int mg, nc, slots, ct, xcap;
};

// Largest token group; for it the most consumer warps (max_consumers, then
// 4 fewer at a time down to 7); for those the deepest ring of code slots
// (4..2, 3..2 with 15 warps) that leaves the activation ring room for two
// entries of the widest projection, else for one; the ring takes the rest
// of the budget.
bool plan_decode(int M, int64_t max_K, DecodePlan *out)
{
    int mg = M;
    while (true) {
        const int nt = (mg + 7) / 8, ct = chunk_tiles(mg);
        const int64_t entry = (mg * (max_K + 64) + 127) / 128 * 128;
        for (int nc = max_consumers(nt); nc >= 7; nc -= 4)
            for (int need = 2; need >= 1; --need)
                for (int s = nc >= 15 ? 3 : 4; s >= 2; --s) {
                    const int64_t rest = kSmemLimit - smem_bytes(nc, s, ct, 0, max_K);
                    const int64_t xcap = rest / 128 * 128;
                    if (xcap >= need * entry) {
                        *out = DecodePlan{mg, nc, s, ct, (int)xcap};
                        return true;
                    }
                }
        if (mg == 1)
            return false;
        mg = mg > 8 ? mg - 8 : mg - 1;
    }
}

cudaError_t launch_plan(const DecodeParams &p, const DecodePlan &g, int grid, int smem,
                        cudaStream_t stream)
{
    // (token tiles, chunk tiles) as chunk_tiles() and max_consumers() give them
    const int nt = (p.mg + 7) / 8;
    if (nt == 1 && g.ct == 7) {
        if (g.nc == 19) return launch_nt<1, 19, 7>(p, grid, smem, stream);
        if (g.nc == 15) return launch_nt<1, 15, 7>(p, grid, smem, stream);
        if (g.nc == 11) return launch_nt<1, 11, 7>(p, grid, smem, stream);
        return launch_nt<1, 7, 7>(p, grid, smem, stream);
    }
    if (nt == 1 && g.ct == 6) {
        if (g.nc == 19) return launch_nt<1, 19, 6>(p, grid, smem, stream);
        if (g.nc == 15) return launch_nt<1, 15, 6>(p, grid, smem, stream);
        if (g.nc == 11) return launch_nt<1, 11, 6>(p, grid, smem, stream);
        return launch_nt<1, 7, 6>(p, grid, smem, stream);
    }
    if (nt == 2 && g.ct == 4) {
        if (g.nc == 15) return launch_nt<2, 15, 4>(p, grid, smem, stream);
        if (g.nc == 11) return launch_nt<2, 11, 4>(p, grid, smem, stream);
        return launch_nt<2, 7, 4>(p, grid, smem, stream);
    }
    if (nt == 3 && g.ct == 6) return launch_nt<3, 7, 6>(p, grid, smem, stream);
    if (nt == 4 && g.ct == 6) return launch_nt<4, 7, 6>(p, grid, smem, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

int quant_launches(int64_t count, int64_t M, int n_big)
{
    return quant_launches_impl(count, M, n_big);
}

cudaError_t launch_quant_own(const DescRecord *table, int count, int64_t M, cudaStream_t stream)
{
    QuantParams q;
    memset(&q, 0, sizeof(q));
    q.table = table;
    q.count = count;
    q.M = (int)M;
    q.own = 1;
    return launch_quant_rows(q, 0, stream);
}

cudaError_t launch_quant_tc(const DescRecord *table, const UnitOrder *order, int n_big, int count,
                            int64_t M, int ntok, uint8_t *ws, int64_t ws_sa_off, cudaStream_t stream)
{
    QuantParams q;
    memset(&q, 0, sizeof(q));
    q.table = table;
    q.count = count;
    q.M = (int)M;
    q.ntok = ntok;
    q.order = order;
    q.ws = ws;
    q.ws_sa_off = ws_sa_off;
    return launch_quant_rows(q, n_big, stream);
}

int decode_launches(int64_t count, int64_t M, int64_t max_K, int n_big)
{
    DecodePlan g{};
    if (!plan_decode((int)M, max_K, &g))
        return 0;
    // quantise (one or two launches) + one decode launch per token group
    return quant_launches(count, M, n_big) + (int)((M + g.mg - 1) / g.mg);
}

cudaError_t launch_decode(const DecodeLaunch &L, uint32_t *err, uint64_t timeout_ns,
                          cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int M = (int)L.M;
    DecodePlan g{};
    if (!plan_decode(M, L.max_K, &g))
        return cudaErrorInvalidValue;

    // Launch 1: quantise every (projection, token) row.
    QuantParams q;
    memset(&q, 0, sizeof(q));
    q.table = L.table;
    if (L.single)
        q.single = *L.single;
    q.count = L.count;
    q.M = M;
    q.ws = L.ws;
    q.ws_sa_off = L.ws_sa_off;
    q.order = L.order;
    e = launch_quant_rows(q, L.n_big, stream);
    if (e != cudaSuccess)
        return e;

    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    if (L.single)
        p.single = *L.single;
    p.count = L.count;
    p.M = M;
    p.total_rb = L.total_rb;
    p.total_cost = L.total_cost;
    p.xs = (int)(L.max_K + 64);
    p.ws = L.ws;
    p.ws_sa_off = L.ws_sa_off;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    p.slots = g.slots;
    p.xcap = g.xcap;
    const int smem = (int)smem_bytes(g.nc, g.slots, g.ct, g.xcap, L.max_K);
    const int64_t grid64 = L.total_rb < sms ? L.total_rb : sms;
    const int grid = (int)(grid64 < 1 ? 1 : grid64);

    for (int m0 = 0; m0 < M; m0 += g.mg) {
        p.m0 = m0;
        p.mg = (M - m0) < g.mg ? (M - m0) : g.mg;
        e = launch_plan(p, g, grid, smem, stream);
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
