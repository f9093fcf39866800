// tw_mid.cu — ternary GEMM for more than 32 tokens with the weights held
// in tensor memory: the 128-row side of tcgen05.mma kind::i8 is a tile of
// ternary codes expanded to int8 {0, 1, 2} (= code + 1) straight into TMEM,
// and the N side is a tile of 64, 96, 128 or 192 int8 token rows (by M)
// loaded by TMA from xq.
//
// What it computes, per projection (per-tensor ternary weights, s =
// 1/mean|W|: "VibeVoice-ASR-BitNet-ONNX" model page, Quantization table; the
// prefill length is the audio frame count plus the prompt, one frame per
// 3200 samples of 24 kHz audio: same page, "Layout"):
//   D[n, m] = sum_k (code[n, k] + 1) * xq[m, k]           (int32, in TMEM)
//   acc     = D - qsum[m],   y[m, n] = ((float)acc * (amax[m] / 127)) * mean|W|
//
// Why weights on the TMEM side: the expanded weights never pass through
// shared memory, which carries only the 2-bit codes and the token tile.  Per
// 128-k stage that is 4 KB of codes and 16 KB of tokens written by TMA and
// read once by the expansion or the MMAs, against 48 KB of operand reads
// plus a 32 KB expanded tile when the weights are the shared-memory operand.
//
// Work unit: one 128-row tile of one projection times one token tile of NT
// tokens (NT = 64, 96, 128 or 192 by M: fewer, fuller units), over all of K; units are claimed from a counter, projections of larger K
// first.  A stage is a pair of 128-column k tiles (one barrier wait and one
// commit of the MMA thread per 8 MMAs):
//   * warp 0 loads the 8 row blocks x 2 k tiles of codes (one 3-D TMA box,
//     k tiles past K read as zero codes) and the two NT x 128 B token tiles
//     (2-D TMA boxes of xq, 128-byte swizzled, tokens past M read as zero)
//     into a ring of L shared-memory stages;
//   * eight expansion warps (two sets of four, one warp per TMEM lane
//     quarter, alternating stages) turn each 16-byte lane slot of the code
//     tile into 16 registers holding code + 1 for 4 consecutive k each, in
//     the natural k order of the MMA's K (each register's 16 source bits
//     come from the word of lane 2(u & 1) + t/2 of the row's quad, fetched
//     with a shuffle), and store them to one of the TMEM A slots of 2 x 32
//     columns (4 up to 128-token units, 2 for 192; tcgen05.st 16x256b: column c
//     of a k tile holds k = 4c .. 4c+3);
//   * warp 1 issues four MMAs of K = 32 per k tile into the unit's
//     accumulator (N = NT columns, one of two) and commits them to the
//     stage's empty barrier, which frees the stage and, four stages later,
//     the A slot;
//   * four epilogue warps (one per lane quarter: 32 weight rows each) read
//     the accumulator 32 tokens at a time (lane = weight row), rescale, and
//     stage the 32 x 32 box in shared memory token by token, then store it
//     with float4 writes: one store instruction covers 4 tokens x 128
//     contiguous bytes of y (measured on B200: one 4-byte store per lane and
//     token left the epilogue at about a third of the MMA rate).
// Every wait is bounded; on a timeout the block stops, drains its copies and
// MMAs, frees its tensor memory and returns.
#include <cstring>

#include "tw_device.cuh"
#include "tw_internal.h"
#include "tw_tc.cuh"

namespace tw {
namespace {

constexpr int kGrpM = kMidGroup;                 // k tiles per stage
constexpr int kRingM = 8;                        // unit-info entries
constexpr int kThreadsM = 14 * 32;
constexpr int kCodeBytesM = 8 * kGrpM * kTileBytes;   // 128 rows x 2 x 128 k = 8 KB
constexpr int kTmemColsM = 512;
constexpr int kMiscM = 2048;

// The shape of a unit of NT tokens (the MMA's N side: 64, 96, 128 or 192):
// the tensor memory holds the two accumulators of NT columns after the A
// slots, which take the rest, at most four (4 slots of a k-tile pair for up
// to 128 tokens, 2 for 192).
template <int NT>
struct MidShape {
    static constexpr int kNTok = NT;
    static constexpr int kFit = (kTmemColsM - 2 * NT) / (32 * kGrpM);
    static constexpr int kASlots = kFit < 4 ? kFit : 4;                     // A slots of kGrpM x 32 columns
    static constexpr int kTokBytes = NT * 128;                               // per k tile
    static constexpr int kStage = kCodeBytesM + kGrpM * kTokBytes;
    static constexpr int kDCol0 = 32 * kGrpM * kASlots;                      // the accumulators
    // int8 x int8 -> int32, K-major, M = 128, N = NT.
    static constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                                       ((128u >> 4) << 24);
    static_assert(NT % 32 == 0 && NT <= 256 && kASlots >= 2, "unit shape");
};
constexpr uint64_t kDrainNsM = 1000000000ull;

struct UnitM {
    int d, rt, tk, live;
};

struct ProjM {
    int64_t N;
    float *y;
    int32_t *acc_out;
    const float *amax;
    const int32_t *qsum;
    float wscale;
    int KT;
};
static_assert(sizeof(ProjM) == 48, "projection cache entry");

struct MidParams {
    const DescRecord *table;
    const UnitOrder *order;   // projections by K, descending, with their first unit
    int count;
    int M;
    int tiles_m;              // token tiles of the unit width
    int64_t total_units;
    uint32_t *ctr;            // [0] claim counter, [1] finished blocks
    WaitCtl ctl;
};

constexpr int kBoxM = 32 * 32 * 4;               // one epilogue warp's staging box
template <int NT, int L>
constexpr int smem_mid(int count)
{
    return 1024 + L * MidShape<NT>::kStage + 4 * kBoxM + kMiscM + (16 + (int)sizeof(ProjM)) * count;
}

__device__ UnitM locate_unit_m(const MidParams &p, const UnitOrder *order, int64_t uid)
{
    int lo = 0, hi = p.count - 1;  // last entry with unit_begin <= uid
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (order[mid].unit_begin <= uid)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int local = (int)(uid - order[lo].unit_begin);
    return UnitM{order[lo].d, local / p.tiles_m, local % p.tiles_m, 1};
}

template <int NT, int L>
__global__ void __launch_bounds__(kThreadsM, 1) k_mid(const __grid_constant__ MidParams p)
{
    using S = MidShape<NT>;
    constexpr int kNTok = S::kNTok, kASlotsM = S::kASlots, kTokBytesM = S::kTokBytes;
    constexpr int kStageM = S::kStage, kDCol0M = S::kDCol0;
    constexpr uint32_t kIdescMid = S::kIdesc;
    static_assert(L >= 2 && L >= kASlotsM, "load stages");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    auto codes_s = [&](int s) { return base + (uint32_t)(s * kStageM); };
    auto tok_s = [&](int s, int j) { return base + (uint32_t)(s * kStageM + kCodeBytesM + j * kTokBytesM); };
    float *boxes = reinterpret_cast<float *>(smem_raw + (base - raw) + L * kStageM);
    uint8_t *misc = smem_raw + (base - raw) + L * kStageM + 4 * kBoxM;
    const uint32_t bar0 = smem_u32(misc);
    const uint32_t b_full = bar0, b_empty = b_full + 8 * L, b_afull = b_empty + 8 * L;
    const uint32_t b_ufull = b_afull + 8 * kASlotsM, b_uempty = b_ufull + 8 * kRingM;
    const uint32_t b_dfull = b_uempty + 8 * kRingM, b_dempty = b_dfull + 16;
    const uint32_t b_drain = b_dempty + 16;
    int *stage_stop = reinterpret_cast<int *>(misc + 1024);
    UnitM *ring = reinterpret_cast<UnitM *>(misc + 1024 + 4 * 32);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 1024 + 4 * 32 + 16 * kRingM);
    int *abort_p = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *abort_flag = abort_p;
    UnitOrder *order_s = reinterpret_cast<UnitOrder *>(misc + kMiscM);
    ProjM *proj_s = reinterpret_cast<ProjM *>(misc + kMiscM + 16 * p.count);
    for (int i = threadIdx.x; i < p.count; i += kThreadsM) {
        order_s[i] = p.order[i];
        const DescRecord &r = p.table[i];
        proj_s[i] = ProjM{r.N, r.y, r.acc_out, r.amax, r.qsum, __ldg(r.wscale), (int)(r.K / kTileK)};
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < L; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, 1);   // the MMA commit of the stage
        }
        for (int a = 0; a < kASlotsM; ++a)
            mbar_init(b_afull + 8 * a, 4);   // the 4 expansion warps of the stage's set
        for (int j = 0; j < kRingM; ++j) {
            mbar_init(b_ufull + 8 * j, 1);
            mbar_init(b_uempty + 8 * j, 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(b_dfull + 8 * b, 1);
            mbar_init(b_dempty + 8 * b, 4);
        }
        mbar_init(b_drain, 1);
        *abort_p = 0;
        fence_barrier_init();
    }
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), kTmemColsM);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            auto resolve = [&](uint32_t uid) {
                return uid < p.total_units ? locate_unit_m(p, order_s, uid) : UnitM{0, 0, 0, 0};
            };
            // claims run two units ahead (the counter's round trip is hidden)
            uint32_t claim1 = atomicAdd(p.ctr, 1u);
            uint32_t claim2 = atomicAdd(p.ctr, 1u);
            for (int j = 0; ok; ++j) {
                const UnitM u = resolve(claim1);
                claim1 = claim2;
                const int ju = j % kRingM;
                if (j >= kRingM &&
                    !mbar_wait(b_uempty + 8 * ju, (uint32_t)((j / kRingM - 1) & 1), p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                ring[ju] = u;
                mbar_arrive(b_ufull + 8 * ju);
                if (!u.live)
                    break;
                claim2 = atomicAdd(p.ctr, 1u);
                const void *tmap_c = p.table[u.d].tmap_codes;   // addresses only
                const void *tmap_x = p.table[u.d].tmap_xq;
                const int KT = proj_s[u.d].KT;
                for (int kt0 = 0; kt0 < KT; kt0 += kGrpM, ++it) {
                    const int s = (int)(it % L);
                    if (it >= L && !mbar_wait(b_empty + 8 * s, (it / L - 1) & 1u, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    stage_stop[s] = 0;
                    const int nk = min(kGrpM, KT - kt0);   // token tiles that exist
                    mbar_arrive_expect_tx(b_full + 8 * s, (uint32_t)(kCodeBytesM + nk * kTokBytesM));
                    tma_load_3d(codes_s(s), tmap_c, 0, kt0, 8 * u.rt, b_full + 8 * s);
                    for (int j = 0; j < nk; ++j)
                        tma_load_2d(tok_s(s, j), tmap_x, (kt0 + j) * 128, u.tk * kNTok, b_full + 8 * s);
                }
            }
            // One stop stage for each expansion set.
            for (int e = 0; e < 2 && ok; ++e, ++it) {
                const int s = (int)(it % L);
                if (it >= L && !mbar_wait(b_empty + 8 * s, (it / L - 1) & 1u, p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                stage_stop[s] = 1;
                mbar_arrive(b_full + 8 * s);
            }
            // Drain: every copy this thread issued lands before the block exits.
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNsM;
            for (uint32_t j = it > (uint32_t)L ? it - L : 0; j < it; ++j)
                mbar_wait(b_full + 8 * (int)(j % L), (j / L) & 1u, drain, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int j = 0; ok; ++j) {
                const int ju = j % kRingM;
                if (!mbar_wait(b_ufull + 8 * ju, (uint32_t)((j / kRingM) & 1), p.ctl, abort_flag))
                    break;
                const UnitM u = ring[ju];
                if (!u.live)
                    break;
                const int buf = j & 1;
                if (j >= 2 &&
                    !mbar_wait(b_dempty + 8 * buf, (uint32_t)((j / 2 - 1) & 1), p.ctl, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d0 = tmem + kDCol0M + (uint32_t)(buf * kNTok);
                const int KT = proj_s[u.d].KT;
                for (int kt0 = 0; kt0 < KT; kt0 += kGrpM, ++it) {
                    // The expansion of this stage waited for its bytes (codes and
                    // tokens) before it arrived here.
                    const int a = (int)(it % kASlotsM);
                    if (!mbar_wait(b_afull + 8 * a, (it / kASlotsM) & 1u, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int s = (int)(it % L);
#pragma unroll
                    for (int j = 0; j < kGrpM; ++j) {
                        if (kt0 + j >= KT)
                            break;   // k tile past K: nothing to add
                        const uint64_t bd = sdesc_k_sw128(tok_s(s, j));
                        const uint32_t acol = tmem + (uint32_t)(32 * (kGrpM * a + j));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // +32 bytes of K = +2 in the address field
                            mma_i8_ts(d0, acol + (uint32_t)(8 * kk), bd + 2 * kk, kIdescMid,
                                      (kt0 > 0 || j > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(b_empty + 8 * s);   // frees stage s, and A slot a for stage it + 4
                }
                if (!ok)
                    break;
                mma_commit(b_dfull + 8 * buf);
            }
            // All MMAs issued by this thread complete before TMEM is freed.
            mma_commit(b_drain);
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNsM;
            mbar_wait(b_drain, 0, drain, nullptr);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        float *box = boxes + (warp - 2) * (kBoxM / 4);   // [32 tokens][32 rows]
        for (int j = 0;; ++j) {
            const int ju = j % kRingM;
            if (!mbar_wait(b_ufull + 8 * ju, (uint32_t)((j / kRingM) & 1), p.ctl, abort_flag))
                break;
            const UnitM u = ring[ju];
            if (!u.live)
                break;
            const ProjM pr = proj_s[u.d];
            const int buf = j & 1;
            const int m_base = u.tk * kNTok;
            // this lane's token of each group of 32: scale and sum(q), loaded
            // before the accumulator is ready
            float sa_l[kNTok / 32];
            int qs_l[kNTok / 32];
#pragma unroll
            for (int c = 0; c < kNTok / 32; ++c) {
                const int m = m_base + 32 * c + lane;
                sa_l[c] = m < p.M ? __fdiv_rn(__ldg(pr.amax + m), 127.f) : 0.f;
                qs_l[c] = m < p.M ? __ldg(pr.qsum + m) : 0;
            }
            if (!mbar_wait(b_dfull + 8 * buf, (uint32_t)((j / 2) & 1), p.ctl, abort_flag))
                break;
            tc_fence_after();
            const uint32_t dq = tmem + kDCol0M + (uint32_t)(buf * kNTok) + ((uint32_t)(32 * quarter) << 16);
            int nvalid = p.M - m_base;
            nvalid = nvalid > kNTok ? kNTok : nvalid;
            const int64_t row0 = (int64_t)u.rt * 128 + 32 * quarter;   // the warp's first row
            // float4 stores need 16-byte aligned rows of y: N a multiple of 4
            const bool vec = (pr.N & 3) == 0 && row0 + 32 <= pr.N;
#pragma unroll 1
            for (int c = 0; c < kNTok / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(dq + 32 * c, v);   // waits for the load
                if (c == kNTok / 32 - 1) {
                    // the accumulator has been read: it may be reused
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(b_dempty + 8 * buf);
                }
                if (32 * c >= nvalid)
                    continue;   // (uniform across the warp)
                // (selected, not indexed: the arrays stay in registers)
                float sa_c = sa_l[0];
                int qs_c = qs_l[0];
#pragma unroll
                for (int i = 1; i < kNTok / 32; ++i)
                    if (c == i) {
                        sa_c = sa_l[i];
                        qs_c = qs_l[i];
                    }
                for (int pass = 0; pass < (pr.acc_out ? 2 : 1); ++pass) {
                    // box[n][lane] = token 32c + n of this lane's row
#pragma unroll
                    for (int n = 0; n < 32; ++n) {
                        const float sa = __shfl_sync(0xffffffffu, sa_c, n);
                        const int qs = __shfl_sync(0xffffffffu, qs_c, n);
                        const int a = (int)v[n] - qs;
                        box[n * 32 + lane] = pass == 0 ? __fmul_rn(__fmul_rn((float)a, sa), pr.wscale)
                                                       : __int_as_float(a);
                    }
                    __syncwarp();
                    float *dst = pass == 0 ? pr.y : reinterpret_cast<float *>(pr.acc_out);
                    const int mmax = nvalid - 32 * c;   // tokens of this box that exist
                    if (vec) {
                        // 8 lanes per token row (128 bytes), 4 tokens per instruction
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int n = 4 * i + (lane >> 3), r4 = 4 * (lane & 7);
                            if (n < mmax)
                                *reinterpret_cast<float4 *>(dst + (int64_t)(m_base + 32 * c + n) * pr.N +
                                                            row0 + r4) =
                                    *reinterpret_cast<const float4 *>(box + n * 32 + r4);
                        }
                    } else {
                        for (int n = 0; n < 32 && n < mmax; ++n)
                            if (row0 + lane < pr.N)
                                dst[(int64_t)(m_base + 32 * c + n) * pr.N + row0 + lane] = box[n * 32 + lane];
                    }
                    __syncwarp();
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(b_uempty + 8 * ju);
        }
    } else {
        // ------------------------------------------------------ expansion
        // Lane (g, t) holds the 16-byte lane slot of rows g, g + 8: word j is
        // row g + 8 (j & 1), k = 64 (j >> 1) + 16 t + 0..15, the code of
        // k0 + 4s + b at bit 8b + 2s.  The 16x256b store gives this lane
        // columns 8u + 2t + (i & 1) of rows g + 8 (i >> 1) (register 4u + i);
        // column c is k = 4c .. 4c + 3, i.e. k0 = 32u + 8t + 4(i & 1), which
        // lives in word 2(u >> 1) + (i >> 1) of lane 4g + 2(u & 1) + (t >> 1),
        // slot s = 2(t & 1) + (i & 1).
        const int quarter = warp & 3, set = (warp - 6) >> 2;
        const int g = lane >> 2, t = lane & 3;
        const uint32_t m3 = 0x03030303u;
        const int sh0 = 4 * (t & 1);   // 2 s for i & 1 == 0
        for (uint32_t it = set;; it += 2) {
            const int s = (int)(it % L);
            // A slot it % kASlotsM is free once the MMAs of stage it - kASlotsM
            // have completed.  That wait comes first: those MMAs follow stage
            // it - L's (kASlotsM <= L), so stage it - L's phase of the load
            // barrier is complete before this set tests it for stage it.  The
            // two sets take alternate stages, and with L odd the previous user
            // of load stage s is the other set: tested first, the barrier
            // could still be in stage it - L's phase, and the parity test
            // would pass at once.
            if (it >= (uint32_t)kASlotsM &&
                !mbar_wait(b_empty + 8 * (int)((it - kASlotsM) % L), ((it - kASlotsM) / L) & 1u, p.ctl,
                           abort_flag))
                break;
            if (!mbar_wait(b_full + 8 * s, (it / L) & 1u, p.ctl, abort_flag))
                break;
            if (stage_stop[s])
                break;
            const uint32_t aslot = it % kASlotsM;
            tc_fence_after();
#pragma unroll
            for (int hj = 0; hj < 2 * kGrpM; ++hj) {
                // row block 2q + h, k tile j of the box (row block by row block)
                const int h = hj & 1, j = hj >> 1;
                const uint4 w = lds128(codes_s(s) + ((2 * quarter + h) * kGrpM + j) * kTileBytes + lane * 16);
                uint32_t r[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int src = 4 * g + 2 * (u & 1) + (t >> 1);
#pragma unroll
                    for (int rh = 0; rh < 2; ++rh) {
                        const int jw = 2 * (u >> 1) + rh;   // uniform across the warp
                        const uint32_t mine = jw == 0 ? w.x : jw == 1 ? w.y : jw == 2 ? w.z : w.w;
                        const uint32_t word = __shfl_sync(0xffffffffu, mine, src);
                        r[4 * u + 2 * rh + 0] = (word >> sh0) & m3;
                        r[4 * u + 2 * rh + 1] = (word >> (sh0 + 2)) & m3;
                    }
                }
                tmem_st16x256b_x4(tmem + 32 * (kGrpM * aslot + j) + ((uint32_t)(32 * quarter + 16 * h) << 16), r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(b_afull + 8 * aslot);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemColsM);
    // The last block to finish clears the counters for the next call.
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.ctr + 1, 1u) == gridDim.x - 1) {
            p.ctr[0] = 0u;
            p.ctr[1] = 0u;
            __threadfence();
        }
    }
}

template <int NT, int L>
cudaError_t launch_mid_l(const MidParams &p, int grid, cudaStream_t stream)
{
    const int smem = smem_mid<NT, L>(p.count);
    cudaError_t e = cudaFuncSetAttribute(k_mid<NT, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    k_mid<NT, L><<<(unsigned)grid, kThreadsM, smem, stream>>>(p);
    return cudaGetLastError();
}

// The deepest ring of load stages that fits beside the caches (fewer stages
// only where every A slot has a load stage of its own).
template <int NT>
cudaError_t launch_mid_nt(const MidParams &p, int grid, cudaStream_t stream)
{
    constexpr int kLimit = 227 * 1024, kA = MidShape<NT>::kASlots;
    if (smem_mid<NT, 5>(p.count) <= kLimit)
        return launch_mid_l<NT, 5>(p, grid, stream);
    if (smem_mid<NT, 4>(p.count) <= kLimit)
        return launch_mid_l<NT, 4>(p, grid, stream);
    if constexpr (kA <= 3)
        if (smem_mid<NT, 3>(p.count) <= kLimit)
            return launch_mid_l<NT, 3>(p, grid, stream);
    if constexpr (kA <= 2)
        if (smem_mid<NT, 2>(p.count) <= kLimit)
            return launch_mid_l<NT, 2>(p, grid, stream);
    return cudaErrorInvalidValue;   // too many projections for the caches
}

}  // namespace

int64_t mid_units(int64_t M, int64_t N)
{
    const int nt = mid_ntok(M);
    return ((N + 127) / 128) * ((M + nt - 1) / nt);
}

cudaError_t launch_mid(const MidLaunch &L, uint32_t *err, uint64_t timeout_ns, cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    MidParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    p.order = L.order;
    p.count = L.count;
    p.M = (int)L.M;
    const int nt = mid_ntok(L.M);
    p.tiles_m = (int)((L.M + nt - 1) / nt);
    p.total_units = L.total_units;
    p.ctr = L.ctr;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    const int64_t grid64 = L.total_units < sms ? L.total_units : sms;
    const int grid = (int)(grid64 < 1 ? 1 : grid64);
    switch (nt) {
    case 64: return launch_mid_nt<64>(p, grid, stream);
    case 96: return launch_mid_nt<96>(p, grid, stream);
    case 192: return launch_mid_nt<192>(p, grid, stream);
    default: return launch_mid_nt<128>(p, grid, stream);
    }
}

}  // namespace tw
