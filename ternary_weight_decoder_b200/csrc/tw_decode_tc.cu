// tw_decode_tc.cu — decode sweep (M <= 32 tokens) on the 5th-generation
// tensor cores: the weights are the 128-row side of tcgen05.mma kind::i8,
// read from tensor memory, and the tokens the N side (8, 16 or 32 columns),
// read from shared memory.
//
// What it computes, per projection: acc = q * codes^T in exact integer
// arithmetic and y = ((float)acc * (amax/127)) * mean|W| (per-tensor ternary
// weights with s = 1/mean|W|: "VibeVoice-ASR-BitNet-ONNX" model page,
// Quantization table; every weight of the 196 projections is read once per
// decode step: "The Paper Says ARM Support" post, "What the model is trying
// to do").  q comes from the quantisation launch of tw_decode.cu, which for
// this path writes each token row already permuted and swizzled (below).
//
// Work unit: one 128-row tile of one projection (8 row blocks of the packed
// layout) over all of K.  Units are claimed from a counter in the scratch,
// projections of larger K first, so that the units left at the end of the
// sweep are the small ones.  A stage is a group of kGrp (six) 128-column k
// tiles (one barrier wait and one commit of the MMA thread per 4 kGrp MMAs:
// measured on B200, the per-stage waits and commits of that single thread,
// not the MMAs, set the pace with one k tile per stage):
//   * warp 0 (producer) loads the 8 row blocks x kGrp k tiles of codes (24 KB)
//     with one 3-D TMA and the kGrp token blocks (N rows x 128 B each) with
//     one bulk copy into a ring of L shared-memory stages (an even number, as
//     many as fit);
//     k tiles past K read as zero codes, which expand to zero weights;
//   * eight expansion warps (two per TMEM lane quarter, alternating stages)
//     turn each 16-byte lane slot of the code tile into 16 registers -- the
//     2-bit slot s of every byte of a word holds codes + 1 of four
//     consecutive k -- and store them to the stage's A slot in tensor memory
//     (tcgen05.st 16x256b): column 8s + 2t + h of lane (row) g or g + 8
//     holds slot s of the word with k = 64h + 16t + 4s .. + 3.  A stage
//     fills one of kASlots A slots of kGrp x 32 columns;
//   * warp 1 waits only for the expansion of the stage (which itself waited
//     for the stage's bytes), issues four MMAs of K = 32 per k tile, one per
//     slot s (columns 8s .. 8s+7), and commits them to the stage's empty
//     barrier, which frees both the shared-memory stage and, kASlots stages
//     later, the A slot;
//   * four epilogue warps (one per lane quarter) read the accumulator, form
//     acc = D - sum(q), exact, then y.
// With 32 tokens the slots are expanded unscaled ((word >> 2s) & 0x03 per
// byte) and every MMA adds into one accumulator D.  With 8 or 16 tokens they
// are expanded with one AND each ((word & (3 << 2s per byte)) is c + 1 times
// 4^s; slot 3, whose 4^3 (c + 1) = 128 does not fit int8, is shifted down
// instead), MMA s adds into accumulator D_s, and the epilogue forms
// D = D_0 + D_1/4 + D_2/16 + D_3 (exact: D_s is a multiple of 4^s).
// The token block pairs position 4c + b of each 128-byte row with the k of
// A column c, so the quantisation launch stores logical k group
// G = 16h + 4t + s of a tile at column c = 8s + 2t + h, and swizzles the
// 16-byte chunks of row n by n mod 8 (the 128-byte swizzle the MMA reads).
//
// Every wait is bounded; on a timeout the block stops, drains its copies and
// MMAs, frees its tensor memory and returns.
#include <cstring>

#include "tw_device.cuh"
#include "tw_internal.h"
#include "tw_tc.cuh"

namespace tw {
namespace {

constexpr int kGrp = kTcGroup;                  // k tiles per stage
constexpr int kRingTc = 8;                      // unit-info entries
constexpr int kMaxStagesTc = 8;                 // shared-memory load stages, at most
constexpr int kThreadsTc = 14 * 32;
constexpr int kCodeStageBytes = 8 * kGrp * kTileBytes;  // 128 rows x kGrp x 128 k
constexpr int kTmemColsTc = 512;

// Tensor-memory plan per token-block width.  32 tokens: one accumulator per
// buffer (every slot's codes expanded unscaled, c + 1 in {0, 1, 2}), so that
// the epilogue reads one accumulator, and three A slots where they fit
// beside it (with four k tiles per stage), so that the expansion stays
// further ahead; 8 or 16 tokens: one accumulator per 2-bit slot (expanded
// with one AND, scaled by 4^s) and two A slots.  Measured on B200 over the
// 196 projections with four k tiles per stage: 138.3 against 144.4 us at 32
// tokens, 117.8 against 119.8 us at 16 for the four-accumulator plan.
template <int NTOK>
struct AccPlan {
    static constexpr bool kOneD = NTOK == 32;
    static constexpr int kASlots = kOneD && 96 * kGrp + 2 * NTOK <= 512 ? 3 : 2;  // A slots of kGrp x 32 columns
    static constexpr int kDCol0 = 32 * kGrp * kASlots;      // the two accumulator buffers
    static constexpr int kDCols = kOneD ? NTOK : 4 * NTOK;  // columns of one buffer
    static_assert(kDCol0 + 2 * kDCols <= 512, "tensor memory");
};
constexpr uint64_t kDrainNsTc = 1000000000ull;

struct UnitInfo {
    int d, rt, KT, live;
};

// The fields of one projection that the block's roles need, copied to shared
// memory once so that no role waits on a global load between units.
struct ProjS {
    int64_t N;
    int64_t ws_xq_off;
    float *y;
    int32_t *acc_out;
    float wscale;
    int KT;
};
static_assert(sizeof(ProjS) == 40, "projection cache entry");

struct TcParams {
    const DescRecord *table;
    const UnitOrder *order;  // projections by K, descending, with their first unit
    int count;
    int M;
    int64_t total_units;
    const uint8_t *ws;       // token blocks at each record's ws_xq_off
    int64_t ws_sa_off;       // amax/127 and sum(q) per projection
    uint32_t *ctr;           // [0] claim counter, [1] finished blocks
    WaitCtl ctl;
};

__device__ __forceinline__ void pdl_wait_tc() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Unit uid -> (projection, 128-row tile), searching the order copied to
// shared memory.
__device__ UnitInfo locate_unit(const TcParams &p, const UnitOrder *order, const ProjS *proj,
                                int64_t uid)
{
    int lo = 0, hi = p.count - 1;  // last entry with unit_begin <= uid
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (order[mid].unit_begin <= uid)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int d = order[lo].d;
    return UnitInfo{d, (int)(uid - order[lo].unit_begin), proj[d].KT, 1};
}

template <int NTOK>
struct Lay_check {
    static constexpr bool ok = (NTOK * 128) % 1024 == 0;   // token blocks stay swizzle-aligned
};

template <int NTOK>
struct TcLayout {
    static constexpr int kBBytes = NTOK * 128;                           // token block
    static constexpr int kBPad = (kBBytes + 1023) / 1024 * 1024;
    static constexpr int kStage = kCodeStageBytes + kGrp * kBPad;
    static constexpr int kMisc = 2048;
    // + the unit order (16 bytes) and the projection cache (40 bytes) per
    // projection after the misc block
    static int smem(int count, int stages) { return 1024 + stages * kStage + kMisc + 56 * count; }
    uint32_t base;
    __device__ uint32_t codes(int s) const { return base + s * kStage; }
    // token block of k tile j (0 .. kGrp - 1) of stage s
    __device__ uint32_t tok(int s, int j = 0) const { return base + s * kStage + kCodeStageBytes + j * kBPad; }
};

// int8 x int8 -> int32, K-major, M = 128, N = NTOK.
template <int NTOK>
__host__ __device__ constexpr uint32_t idesc_tc()
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NTOK >> 3) << 17) | ((128u >> 4) << 24);
}

template <int NTOK>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&v)[NTOK])
{
    if constexpr (NTOK == 8)
        tmem_ld8(taddr, v);
    else if constexpr (NTOK == 16)
        tmem_ld16(taddr, v);
    else
        tmem_ld32_nowait(taddr, v);
}

// L shared-memory stages (4 .. kMaxStagesTc).  Stage counters are 32-bit:
// a block streams at most a few thousand stages per call.
template <int NTOK, int L>
__global__ void __launch_bounds__(kThreadsTc, 1) k_decode_tc(const __grid_constant__ TcParams p)
{
    using AP = AccPlan<NTOK>;
    constexpr int kASlots = AP::kASlots, kDCol0 = AP::kDCol0;
    static_assert(L >= kASlots && L <= kMaxStagesTc && L % 2 == 0, "load stages");
    static_assert(Lay_check<NTOK>::ok, "token blocks");
    using Lay = TcLayout<NTOK>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const Lay lay{base};
    uint8_t *misc = smem_raw + (base - raw) + L * Lay::kStage;
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
    const uint32_t bar0 = smem_u32(bars);
    // full/empty: per load stage; afull: per A slot
    const uint32_t b_full = bar0, b_empty = b_full + 8 * L, b_afull = b_empty + 8 * L;
    const uint32_t b_ufull = b_afull + 8 * kASlots, b_uempty = b_ufull + 8 * kRingTc;
    const uint32_t b_dfull = b_uempty + 8 * kRingTc, b_dempty = b_dfull + 16;
    const uint32_t b_drain = b_dempty + 16;
    int *stage_stop = reinterpret_cast<int *>(misc + 1024);
    UnitInfo *ring = reinterpret_cast<UnitInfo *>(misc + 1024 + 4 * kMaxStagesTc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 1024 + 4 * kMaxStagesTc + 16 * kRingTc);
    int *abort_p = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *abort_flag = abort_p;
    UnitOrder *order_s = reinterpret_cast<UnitOrder *>(misc + Lay::kMisc);
    ProjS *proj_s = reinterpret_cast<ProjS *>(misc + Lay::kMisc + 16 * p.count);
    for (int i = threadIdx.x; i < p.count; i += kThreadsTc) {
        order_s[i] = p.order[i];
        const DescRecord &r = p.table[i];
        proj_s[i] = ProjS{r.N, r.ws_xq_off, r.y, r.acc_out, __ldg(r.wscale), (int)(r.K / kTileK)};
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < L; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, 1);   // the MMA commit of the stage
        }
        for (int a = 0; a < kASlots; ++a)
            mbar_init(b_afull + 8 * a, 4);   // the 4 expansion warps of the stage's set
        for (int j = 0; j < kRingTc; ++j) {
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
        tmem_alloc(smem_u32(tmem_slot), kTmemColsTc);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true, tokens_ready = false;
            // Token blocks of the stages issued before launch 1 has finished:
            // the codes of the first stages stream while it still quantises.
            const uint8_t *pend_src[L];
            int pend_s[L], pend_n[L];
            int npend = 0;
            auto flush_tokens = [&]() {
                pdl_wait_tc();
                tokens_ready = true;
                for (int i = 0; i < npend; ++i)
                    bulk_g2s(lay.tok(pend_s[i]), pend_src[i], (uint32_t)(pend_n[i] * Lay::kBBytes),
                             b_full + 8 * pend_s[i]);
                npend = 0;
            };
            // Claims run two units ahead, so that the counter's round trip is
            // hidden behind the streaming of the current unit.
            auto resolve = [&](uint32_t uid) {
                return uid < p.total_units ? locate_unit(p, order_s, proj_s, uid)
                                           : UnitInfo{0, 0, 0, 0};
            };
            uint32_t claim1 = atomicAdd(p.ctr, 1u);
            uint32_t claim2 = atomicAdd(p.ctr, 1u);
            for (int j = 0; ok; ++j) {
                const UnitInfo u = resolve(claim1);
                claim1 = claim2;
                const int ju = j % kRingTc;
                if (j >= kRingTc &&
                    !mbar_wait(b_uempty + 8 * ju, (uint32_t)((j / kRingTc - 1) & 1), p.ctl, abort_flag)) {
                    ok = false;
                    break;
                }
                ring[ju] = u;
                mbar_arrive(b_ufull + 8 * ju);
                if (!u.live)
                    break;
                claim2 = atomicAdd(p.ctr, 1u);
                const void *tmap = p.table[u.d].tmap_codes;   // address only
                const uint8_t *tok_src = p.ws + proj_s[u.d].ws_xq_off;
                for (int kt0 = 0; kt0 < u.KT; kt0 += kGrp, ++it) {
                    const int s = (int)(it % L);
                    if (it >= L &&
                        !mbar_wait(b_empty + 8 * s, (it / L - 1) & 1u, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    stage_stop[s] = 0;
                    const int nk = min(kGrp, u.KT - kt0);   // token blocks that exist
                    mbar_arrive_expect_tx(b_full + 8 * s,
                                          (uint32_t)(kCodeStageBytes + nk * Lay::kBBytes));
                    tma_load_3d(lay.codes(s), tmap, 0, kt0, 8 * u.rt, b_full + 8 * s);
                    const uint8_t *src = tok_src + (int64_t)kt0 * Lay::kBBytes;
                    if (tokens_ready) {
                        bulk_g2s(lay.tok(s), src, (uint32_t)(nk * Lay::kBBytes), b_full + 8 * s);
                    } else {
                        pend_src[npend] = src;
                        pend_n[npend] = nk;
                        pend_s[npend] = s;
                        if (++npend == L)
                            flush_tokens();   // before any stage is waited on again
                    }
                }
            }
            if (!tokens_ready)
                flush_tokens();
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
            drain.timeout_ns = kDrainNsTc;
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
                const int ju = j % kRingTc;
                if (!mbar_wait(b_ufull + 8 * ju, (uint32_t)((j / kRingTc) & 1), p.ctl, abort_flag))
                    break;
                const UnitInfo u = ring[ju];
                if (!u.live)
                    break;
                const int buf = j & 1;
                if (j >= 2 &&
                    !mbar_wait(b_dempty + 8 * buf, (uint32_t)((j / 2 - 1) & 1), p.ctl, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d0 = tmem + kDCol0 + (uint32_t)(buf * AP::kDCols);
                for (int kt0 = 0; kt0 < u.KT; kt0 += kGrp, ++it) {
                    // The expansion of this stage waited for its bytes (codes and
                    // token blocks) before it arrived here.
                    const int a = (int)(it % kASlots);
                    if (!mbar_wait(b_afull + 8 * a, (it / kASlots) & 1u, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int s = (int)(it % L);
                    // Descriptors of the stage: k tile j's token block is kBPad
                    // bytes after the previous one; +32 bytes of K = +2 in the
                    // address field.  A full group runs without a test per
                    // k tile (measured: 130.1 -> 128.0 us at 20 tokens).
                    const uint64_t bd0 = sdesc_k_sw128(lay.tok(s, 0));
                    const uint32_t acol0 = tmem + (uint32_t)(32 * kGrp * a);
                    const uint32_t first = kt0 > 0 ? 1u : 0u;
                    auto mma_tile = [&](int j) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t d = AP::kOneD ? d0 : d0 + (uint32_t)(kk * NTOK);
                            const uint32_t acc_in = j > 0 || (AP::kOneD && kk > 0) ? 1u : first;
                            mma_i8_ts(d, acol0 + (uint32_t)(32 * j + 8 * kk),
                                      bd0 + (uint64_t)((Lay::kBPad >> 4) * j + 2 * kk), idesc_tc<NTOK>(),
                                      acc_in);
                        }
                    };
                    if (kt0 + kGrp <= u.KT) {
#pragma unroll
                        for (int j = 0; j < kGrp; ++j)
                            mma_tile(j);
                    } else {
#pragma unroll
                        for (int j = 0; j < kGrp; ++j) {
                            if (kt0 + j >= u.KT)
                                break;   // k tiles past K (zero codes): nothing to add
                            mma_tile(j);
                        }
                    }
                    mma_commit(b_empty + 8 * s);   // frees stage s, and A slot a for stage it + 2
                }
                if (!ok)
                    break;
                mma_commit(b_dfull + 8 * buf);
            }
            // All MMAs issued by this thread complete before TMEM is freed.
            mma_commit(b_drain);
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNsTc;
            mbar_wait(b_drain, 0, drain, nullptr);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        for (int j = 0;; ++j) {
            const int ju = j % kRingTc;
            if (!mbar_wait(b_ufull + 8 * ju, (uint32_t)((j / kRingTc) & 1), p.ctl, abort_flag))
                break;
            const UnitInfo u = ring[ju];
            if (!u.live)
                break;
            const ProjS pr = proj_s[u.d];
            const int64_t N = pr.N;
            float *const y = pr.y;
            int32_t *const acc_out = pr.acc_out;
            const float wscale = pr.wscale;
            const int buf = j & 1;
            if (!mbar_wait(b_dfull + 8 * buf, (uint32_t)((j / 2) & 1), p.ctl, abort_flag))
                break;
            tc_fence_after();
            // The scales of launch 1: read only after the accumulator is
            // complete, which is after the producer waited for launch 1.
            const uint8_t *info = p.ws + p.ws_sa_off + 256 * (int64_t)u.d;
            const float sa_l = lane < p.M ? reinterpret_cast<const float *>(info)[lane] : 0.f;
            const int qs_l = lane < p.M ? reinterpret_cast<const int *>(info + 128)[lane] : 0;
            const uint32_t dq = tmem + kDCol0 + (uint32_t)(buf * AP::kDCols) + ((uint32_t)(32 * quarter) << 16);
            int acc[NTOK];
            {
                uint32_t v[NTOK];
                tmem_ld_n<NTOK>(dq, v);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NTOK; ++n)
                    acc[n] = (int)v[n];
            }
            if constexpr (!AP::kOneD) {
                uint32_t v[NTOK];
                tmem_ld_n<NTOK>(dq + NTOK, v);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NTOK; ++n)
                    acc[n] += (int)v[n] >> 2;
                tmem_ld_n<NTOK>(dq + 2 * NTOK, v);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NTOK; ++n)
                    acc[n] += (int)v[n] >> 4;
                tmem_ld_n<NTOK>(dq + 3 * NTOK, v);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NTOK; ++n)
                    acc[n] += (int)v[n];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(b_dempty + 8 * buf);
            const int64_t row = (int64_t)u.rt * 128 + 32 * quarter + lane;
#pragma unroll
            for (int n = 0; n < NTOK; ++n) {
                const float sa = __shfl_sync(0xffffffffu, sa_l, n);
                const int qs = __shfl_sync(0xffffffffu, qs_l, n);
                if (n < p.M && row < N) {
                    const int v = acc[n] - qs;
                    y[(int64_t)n * N + row] = __fmul_rn(__fmul_rn((float)v, sa), wscale);
                    if (acc_out)
                        acc_out[(int64_t)n * N + row] = v;
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(b_uempty + 8 * ju);
        }
    } else {
        // ------------------------------------------------------ expansion
        const int quarter = warp & 3, set = (warp - 6) >> 2;
        const uint32_t m = 0x03030303u;
        for (uint32_t it = set;; it += 2) {
            const int s = (int)(it % L);
            if (!mbar_wait(b_full + 8 * s, (it / L) & 1u, p.ctl, abort_flag))
                break;
            if (stage_stop[s])
                break;
            // A slot it % kASlots is free once the MMAs of stage it - kASlots
            // have completed.
            if (it >= (uint32_t)kASlots &&
                !mbar_wait(b_empty + 8 * (int)((it - kASlots) % L), ((it - kASlots) / L) & 1u, p.ctl,
                           abort_flag))
                break;
            const uint32_t aslot = it % kASlots;
            tc_fence_after();
#pragma unroll
            for (int hj = 0; hj < 2 * kGrp; ++hj) {
                // k tile j, row block 2q + h of the stage's box (laid out row
                // block by row block, k tiles inside): lane slot words (row g,
                // k 16t..), (row g+8, same k), (row g, k 64+16t..), (row g+8, same k)
                const int h = hj & 1, j = hj >> 1;
                const uint4 w = lds128(lay.codes(s) + ((2 * quarter + h) * kGrp + j) * kTileBytes + lane * 16);
                uint32_t r[16];
                if constexpr (AP::kOneD) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        r[4 * u + 0] = (w.x >> (2 * u)) & m;
                        r[4 * u + 1] = (w.z >> (2 * u)) & m;
                        r[4 * u + 2] = (w.y >> (2 * u)) & m;
                        r[4 * u + 3] = (w.w >> (2 * u)) & m;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 3; ++u) {
                        const uint32_t mu = m << (2 * u);
                        r[4 * u + 0] = w.x & mu;
                        r[4 * u + 1] = w.z & mu;
                        r[4 * u + 2] = w.y & mu;
                        r[4 * u + 3] = w.w & mu;
                    }
                    r[12] = (w.x >> 6) & m;
                    r[13] = (w.z >> 6) & m;
                    r[14] = (w.y >> 6) & m;
                    r[15] = (w.w >> 6) & m;
                }
                tmem_st16x256b_x4(tmem + 32 * (kGrp * aslot + j) + ((uint32_t)(32 * quarter + 16 * h) << 16), r);
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
        tmem_dealloc(tmem, kTmemColsTc);
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

template <int NTOK, int L>
cudaError_t launch_tc_l(const TcParams &p, int grid, cudaStream_t stream)
{
    const int smem = TcLayout<NTOK>::smem(p.count, L);
    cudaError_t e = cudaFuncSetAttribute(k_decode_tc<NTOK, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    // Programmatic dependent launch: the codes stream while launch 1 runs.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode_tc<NTOK, L>, p);
}

// The deepest ring of load stages that fits in shared memory beside the
// per-projection caches (more stages keep more code bytes in flight).
template <int NTOK>
cudaError_t launch_tc(const TcParams &p, int grid, cudaStream_t stream)
{
    constexpr int kLimit = 227 * 1024;
    if (TcLayout<NTOK>::smem(p.count, 8) <= kLimit)
        return launch_tc_l<NTOK, 8>(p, grid, stream);
    if (TcLayout<NTOK>::smem(p.count, 6) <= kLimit)
        return launch_tc_l<NTOK, 6>(p, grid, stream);
    if (TcLayout<NTOK>::smem(p.count, 4) <= kLimit)
        return launch_tc_l<NTOK, 4>(p, grid, stream);
    return cudaErrorInvalidValue;   // too many projections for the caches
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeTcLaunch &L, uint32_t *err, uint64_t timeout_ns,
                             cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    e = launch_quant_tc(L.table, L.order, L.n_big, L.count, L.M, tc_tokens(L.M), L.ws, L.ws_sa_off,
                        stream);
    if (e != cudaSuccess)
        return e;
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    p.order = L.order;
    p.count = L.count;
    p.M = (int)L.M;
    p.total_units = L.total_units;
    p.ws = L.ws;
    p.ws_sa_off = L.ws_sa_off;
    p.ctr = L.ctr;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    const int64_t grid64 = L.total_units < sms ? L.total_units : sms;
    const int grid = (int)(grid64 < 1 ? 1 : grid64);
    switch (tc_tokens(L.M)) {
    case 8: return launch_tc<8>(p, grid, stream);
    case 16: return launch_tc<16>(p, grid, stream);
    default: return launch_tc<32>(p, grid, stream);
    }
}

}  // namespace tw
