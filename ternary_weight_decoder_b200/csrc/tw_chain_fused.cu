// tw_chain_fused.cu — the decoder-layer chain as one persistent kernel per
// group of up to 8 tokens: every layer's four dependent stages (q/k/v, o,
// gate/up, down) with grid-wide barriers between them, the activation
// quantisation, the rescale, the attention stand-in, both residual adds and
// SiLU(gate) * up fused into the stages.  (The decoder layer of the
// Qwen2.5-1.5B LM: "VibeVoice-ASR-BitNet-ONNX" model page, "Layout"; every
// weight is read once per token: "The Paper Says ARM Support" post, "What
// the model is trying to do".)
//
// Launch: cooperative, one CTA per SM (all co-resident, so the barriers
// cannot deadlock), NW warps each.
//
// A stage's work is split into units of one 16-row block x up to 6 code
// tiles (768 k) of one projection -- split-K, so that the down projection's
// 96 long row blocks spread over every warp of the grid.  The CTAs take
// equal ranges of units, their warps every NW-th unit.  Each warp keeps a
// ring of S slots that it fills with 1-D bulk copies of its next units'
// codes, across stage boundaries: the weights do not depend on the
// activations, so the code stream runs ahead while the grid waits.  A unit's
// partial sums D = sum_k (c + 1) q are added into an int32 buffer of the
// stage with integer atomics (exact in any order).
//
// Stage s's prologue (every CTA, every thread, after the barrier): read the
// previous stage's sums, rescale them exactly as the single-projection
// epilogue does, y = ((float)(D - sum q) * (amax/127)) * wscale, apply the
// step between the stages -- q/k/v -> a = v repeated per query-head group;
// o -> h1 = h + o; gate/up -> SiLU(g) * u; down -> h' = h1 + d -- and
// quantise the result per token (amax, 127/amax, rint) into shared memory
// for the stage's MMAs.  Each CTA computes the whole input rows (they are a
// few KB at decode sizes) but writes only its slice of the materialised
// buffers (q, k, v, a, o, h1, g, u, act, d, h and any acc_out).  The sums
// live in kChainSumBufs = 4 rotating buffers: stage s adds into buffer
// s mod 4; stage s + 1 reads it (its prologue, and its materialisation,
// which runs after its units, between its arrival at the barrier and its
// wait); stage s clears the buffer of s + 1 before it arrives at its
// barrier -- so every buffer is zero before the first atomic reaches it,
// and none is cleared while a CTA still materialises from it.
//
// Every value is computed with the same fp32 operations as the unfused
// chain (the same rounding), so the two give the same bytes.  Every wait is
// bounded: a barrier or ring wait that expires sets the timeout bit, stops
// the block and drains its copies.
#include <cstring>

#include "tw_device.cuh"
#include "tw_gemv.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kNW = 16;                    // warps per CTA (all consume and quantise)
constexpr int kCT = kChainChunk;           // code tiles per unit (one ring slot)
constexpr int kS = 3;                      // ring slots per warp
constexpr int kThreadsCh = kNW * 32;
constexpr int kSlotBytes = kCT * kTileBytes;
constexpr uint64_t kDrainNsCh = 1000000000ull;
// A stage input row of up to kXR float4 per thread (K <= 10240) for up to
// kRegTokens tokens stays in registers between the amax and the
// quantisation passes; each pass then issues all its loads at once.  (Two
// tokens spill registers of the 512-thread CTA.)
constexpr int kXR = 5;
constexpr int kRegTokens = 1;
// The down projection's input as read back by the quantisation: SiLU(g) * u
// is computed once, by the CTA whose slice of `act` holds it (materialise),
// and after a grid-wide barrier read by every CTA (measured on B200: every
// CTA computing the whole row took 7 us per down stage).
constexpr int kStageDownAct = 4;

struct ChainParams {
    const ChainPlanHeader *plan;
    uint8_t *ws;
    int m0, mg;                 // token group [m0, m0 + mg)
    int xstride;                // bytes per activation row in shared memory (max_K + 64)
    int unit_cache;             // the stages' unit fields are copied to shared memory
    WaitCtl ctl;
};

// What a warp's walk over its units needs of each stage -- this CTA's range
// [lo, hi) of the stage's units among them -- computed once per stage and
// kept in shared memory when it fits (measured on B200: read from the plan
// in global memory with two 64-bit divisions per step, a warp's step from
// its last unit of a stage to its first of the next took 0.6-1 us, on every
// stage's critical path).
struct UnitS {
    int lo, hi, nch, KT;
    int rb_off[4];              // first row block of each projection; past nproj: the total
    const uint8_t *packed[3];
    int nproj, pad;
};
static_assert(sizeof(UnitS) == 64, "unit cache entry");

__device__ __forceinline__ UnitS unit_fields(const ChainStagePlan *st)
{
    UnitS u;
    const int64_t units = st->units;
    u.lo = (int)(units * blockIdx.x / gridDim.x);
    u.hi = (int)(units * (blockIdx.x + 1) / gridDim.x);
    u.nch = st->nch;
    u.KT = st->K / kTileK;
    u.nproj = st->nproj;
    // entries past the stage's projections hold the total, so where() never
    // picks them
    for (int q = 0; q < 3; ++q) {
        u.rb_off[q] = q < u.nproj ? (int)st->proj[q].rb_off : (int)st->rb_total;
        u.packed[q] = st->proj[q].packed;
    }
    u.rb_off[3] = (int)st->rb_total;
    u.pad = 0;
    return u;
}

__device__ __forceinline__ const ChainStagePlan *stage_of(const ChainPlanHeader *h, int s)
{
    return reinterpret_cast<const ChainStagePlan *>(h + 1) + s;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add_u32(uint32_t *p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" : : "l"(p), "r"(v) : "memory");
}

// Grid-wide barrier number `k` (1, 2, ...): every CTA's writes before it are
// visible to every CTA after it.  ctr[0] counts arrivals over the whole call;
// after __syncthreads thread 0 adds its CTA's arrival with release semantics
// (which carry the CTA's writes ordered before it by the block barrier) and
// polls the count with acquire loads until all k * gridDim.x arrivals are in.
// The release and acquire replace two full fences per CTA.  False when the
// wait timed out (the block must stop).
// The barrier in two halves: the arrival, then -- after work that needs no
// other CTA's -- the wait.
__device__ __forceinline__ void grid_arrive(uint32_t *ctr)
{
    __syncthreads();
    if (threadIdx.x == 0)
        red_release_add_u32(ctr, 1u);
}

__device__ bool grid_wait(uint32_t *ctr, uint32_t k, const ChainParams &p, volatile int *abort_flag)
{
    if (threadIdx.x == 0) {
        const uint32_t target = k * gridDim.x;
        if (!*abort_flag && ld_acquire_u32(ctr) < target) {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u32(ctr) < target) {
                if (*abort_flag)
                    break;
                if (globaltimer_ns() - t0 > p.ctl.timeout_ns) {
                    atomicOr(p.ctl.err, EFLAG_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
            }
        }
    }
    __syncthreads();
    return !*abort_flag;
}

__device__ __forceinline__ bool grid_barrier(uint32_t *ctr, uint32_t k, const ChainParams &p,
                                             volatile int *abort_flag)
{
    grid_arrive(ctr);
    return grid_wait(ctr, k, p, abort_flag);
}

// A warp's walk over its work units, stage after stage.  Its fields are
// scalars, indexed by selection, so that it stays in registers (measured on
// B200: with arrays indexed by the projection it lived in local memory,
// which the large shared-memory carve-out leaves no L1 for, and each step
// paid L2 round trips).
struct UnitIter {
    int s, n_stages;
    int u, hi;                  // current unit, end of this CTA's range in stage s
    int nch, KT, nproj;
    int rb1, rb2;               // first row block of projections 1 and 2 (the total past nproj)
    const uint8_t *packed0, *packed1, *packed2;
    bool valid;
    const UnitS *cache;         // the stages' unit fields in shared memory, or null

    __device__ void enter(const ChainPlanHeader *h, int stage, int w)
    {
        valid = false;
        for (s = stage; s < n_stages; ++s) {
            const UnitS f = cache ? cache[s] : unit_fields(stage_of(h, s));
            hi = f.hi;
            u = f.lo + w;
            if (u < hi) {
                nch = f.nch;
                KT = f.KT;
                nproj = f.nproj;
                rb1 = f.rb_off[1];
                rb2 = f.rb_off[2];
                packed0 = f.packed[0];
                packed1 = f.packed[1];
                packed2 = f.packed[2];
                valid = true;
                return;
            }
        }
    }
    __device__ void next(const ChainPlanHeader *h, int w)
    {
        u += kNW;
        if (u >= hi)
            enter(h, s + 1, w);
    }
    // (projection, row block in it, first tile, tiles) of the current unit
    __device__ void where(int &q, int &rbl, int &kt0, int &n) const
    {
        const int rbg = u / nch, kc = u - rbg * nch;
        q = rbg >= rb1 ? (rbg >= rb2 ? 2 : 1) : 0;
        rbl = rbg - (q == 0 ? 0 : q == 1 ? rb1 : rb2);
        kt0 = kc * kCT;
        n = min(kCT, KT - kt0);
    }
    __device__ void issue(uint32_t dst, uint32_t bar) const
    {
        int q, rbl, kt0, n;
        where(q, rbl, kt0, n);
        const uint8_t *src = (q == 0 ? packed0 : q == 1 ? packed1 : packed2) +
                             ((int64_t)rbl * KT + kt0) * (int64_t)kTileBytes;
        mbar_arrive_expect_tx(bar, (uint32_t)(n * kTileBytes));
        bulk_g2s(dst, src, (uint32_t)(n * kTileBytes), bar);
    }
};

__device__ __forceinline__ float rescale1(int D, int qs, float sa, float ws)
{
    return __fmul_rn(__fmul_rn((float)(D - qs), sa), ws);
}

__device__ __forceinline__ float silu_mul1(float z, float u)
{
    return __fmul_rn(__fdiv_rn(z, __fadd_rn(1.0f, expf(-z))), u);
}

// The stage input x(m, 4i .. 4i+3) of the prologue of stage kind `kind`
// (layer's first stage when first_layer), from the previous stage's sums
// `sum` (row stride prev->ntot) with the previous input's scales.  The
// helpers below also return the materialised values the slice writers need.
struct Prev {
    const int32_t *sum;         // previous stage's sums (token-major, ntot per row)
    int64_t ntot;
    const ChainStagePlan *st;   // previous stage
    const float *sa;            // its input's amax/127 per token (shared memory)
    const int *qs;              // its input's sum(q) per token (shared memory)
    const float *ws;            // its projections' wscale (shared memory)
};

__device__ __forceinline__ int4 ldcg4i(const int32_t *p) { return __ldcg(reinterpret_cast<const int4 *>(p)); }
__device__ __forceinline__ float4 ldcg4f(const float *p) { return __ldcg(reinterpret_cast<const float4 *>(p)); }

// y (fp32) of column j .. j+3 of projection q of the previous stage, token m.
__device__ __forceinline__ float4 prev_y4(const Prev &P, int q, int m, int64_t j)
{
    const float ws = P.ws[q];
    const int4 D = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[q].noff + j);
    return make_float4(rescale1(D.x, P.qs[m], P.sa[m], ws), rescale1(D.y, P.qs[m], P.sa[m], ws),
                       rescale1(D.z, P.qs[m], P.sa[m], ws), rescale1(D.w, P.qs[m], P.sa[m], ws));
}

__device__ __forceinline__ float4 add4(float4 a, float4 b)
{
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}

// x of stage `kind` at token m (chain row m0 + m), columns 4i .. 4i + 3.
__device__ __forceinline__ float4 stage_x4(const ChainPlanHeader *h, int kind, bool first_layer,
                                           const Prev &P, int m, int mrow, int64_t i)
{
    const int64_t k = 4 * i;
    switch (kind) {
    case kStageQKV:
        if (first_layer)
            return ldcg4f(h->h + mrow * h->hidden + k);
        // h' = h1 + d of the previous layer
        return add4(ldcg4f(h->h1 + mrow * h->hidden + k), prev_y4(P, 0, m, k));
    case kStageO: {
        // a = v, each KV head repeated for the query heads of its group
        const int hd = (int)h->head_dim, group = (int)(h->hidden / h->kv_dim);
        const int head = (int)k / hd, c = (int)k - head * hd;
        return prev_y4(P, 2, m, (head / group) * h->head_dim + c);
    }
    case kStageGU:
        return add4(ldcg4f(h->h + mrow * h->hidden + k), prev_y4(P, 0, m, k));
    case kStageDownAct:
        return ldcg4f(h->act + mrow * h->inter + k);
    default: {   // kStageDown: SiLU(g) * u
        const float4 g = prev_y4(P, 0, m, k);
        const float4 u = prev_y4(P, 1, m, k);
        return make_float4(silu_mul1(g.x, u.x), silu_mul1(g.y, u.y), silu_mul1(g.z, u.z),
                           silu_mul1(g.w, u.w));
    }
    }
}

// The same value as stage_x4, in two steps: stage_raw issues the loads
// (up to two 16-byte words: a = h, h1 or the sums of projection 0; b = the
// sums of the projection the step reads), stage_val computes from them.  A
// caller that loads all its elements before computing any has one L2
// round trip in flight instead of one per element.
__device__ __forceinline__ void stage_raw(const ChainPlanHeader *h, int kind, bool first_layer,
                                          const Prev &P, int m, int mrow, int64_t i, int4 &a, int4 &b)
{
    const int64_t k = 4 * i;
    switch (kind) {
    case kStageQKV:
        if (first_layer) {
            a = ldcg4i(reinterpret_cast<const int32_t *>(h->h + mrow * h->hidden + k));
        } else {
            a = ldcg4i(reinterpret_cast<const int32_t *>(h->h1 + mrow * h->hidden + k));
            b = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[0].noff + k);
        }
        break;
    case kStageO: {
        const int hd = (int)h->head_dim, group = (int)(h->hidden / h->kv_dim);
        const int head = (int)k / hd, c = (int)k - head * hd;
        b = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[2].noff + (head / group) * h->head_dim + c);
        break;
    }
    case kStageGU:
        a = ldcg4i(reinterpret_cast<const int32_t *>(h->h + mrow * h->hidden + k));
        b = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[0].noff + k);
        break;
    case kStageDownAct:
        a = ldcg4i(reinterpret_cast<const int32_t *>(h->act + mrow * h->inter + k));
        break;
    default:
        a = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[0].noff + k);
        b = ldcg4i(P.sum + (int64_t)m * P.ntot + P.st->proj[1].noff + k);
        break;
    }
}

__device__ __forceinline__ float4 rescale4(int4 D, const Prev &P, int q, int m)
{
    const float ws = P.ws[q];
    return make_float4(rescale1(D.x, P.qs[m], P.sa[m], ws), rescale1(D.y, P.qs[m], P.sa[m], ws),
                       rescale1(D.z, P.qs[m], P.sa[m], ws), rescale1(D.w, P.qs[m], P.sa[m], ws));
}

__device__ __forceinline__ float4 as_f4(int4 a)
{
    return make_float4(__int_as_float(a.x), __int_as_float(a.y), __int_as_float(a.z), __int_as_float(a.w));
}

__device__ __forceinline__ float4 stage_val(int kind, bool first_layer, const Prev &P, int m, int4 a,
                                            int4 b)
{
    switch (kind) {
    case kStageQKV:
        return first_layer ? as_f4(a) : add4(as_f4(a), rescale4(b, P, 0, m));
    case kStageO:
        return rescale4(b, P, 2, m);
    case kStageGU:
        return add4(as_f4(a), rescale4(b, P, 0, m));
    case kStageDownAct:
        return as_f4(a);
    default: {
        const float4 g = rescale4(a, P, 0, m), u = rescale4(b, P, 1, m);
        return make_float4(silu_mul1(g.x, u.x), silu_mul1(g.y, u.y), silu_mul1(g.z, u.z),
                           silu_mul1(g.w, u.w));
    }
    }
}

__device__ __forceinline__ uint32_t quant4c(float4 v, float scale, bool zero, int &sum)
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

// This CTA's share [lo, hi) of n items: [n c / G, n (c + 1) / G).  In
// 32-bit arithmetic when n G fits (a 64-bit division is a long call on the
// GPU, and these sit on every stage's path; measured on B200: about 0.3 us
// per stage for the two of the sum-buffer clearing alone).
__device__ __forceinline__ void cta_share(int64_t n, int64_t &lo, int64_t &hi)
{
    const uint32_t G = gridDim.x, c = blockIdx.x;
    if (n >= 0 && n * (int64_t)G < ((int64_t)1 << 32)) {
        const uint32_t n32 = (uint32_t)n;
        lo = n32 * c / G;
        hi = n32 * (c + 1) / G;
    } else {
        lo = n * c / G;
        hi = n * (c + 1) / G;
    }
}

// Write this CTA's slice of an [mg x width] materialised buffer: element e
// of the slice has value fn(m, j) for m = e / width, j = e % width (width a
// multiple of 4; written 4 at a time) -- by threads tid = 0 .. nt - 1 of a
// group of the CTA's warps.
template <class F>
__device__ __forceinline__ void write_slice(float *dst, int64_t width, int mg, int m0, int tid, int nt,
                                            F fn)
{
    const int64_t n4 = (int64_t)mg * width / 4;
    int64_t lo, hi;
    cta_share(n4, lo, hi);
    const bool narrow = n4 < ((int64_t)1 << 31);   // (32-bit index arithmetic)
    const uint32_t w4 = (uint32_t)(width / 4);
    for (int64_t e = lo + tid; e < hi; e += nt) {
        const int m = narrow ? (int)((uint32_t)e / w4) : (int)(e / (width / 4));
        const int64_t j = 4 * (e - (int64_t)m * (width / 4));
        *reinterpret_cast<float4 *>(dst + (int64_t)(m0 + m) * width + j) = fn(m, j);
    }
}

// This CTA's slice of the previous stage's integer outputs into acc_out.
__device__ __forceinline__ void write_acc_slice(const Prev &P, int q, int mg, int m0, int tid, int nt)
{
    const ChainProj &pr = P.st->proj[q];
    if (!pr.acc_out)
        return;
    const int64_t width = pr.N;
    const int64_t n = (int64_t)mg * width;
    int64_t lo, hi;
    cta_share(n, lo, hi);
    const bool narrow = n < ((int64_t)1 << 31);
    for (int64_t e = lo + tid; e < hi; e += nt) {
        const int m = narrow ? (int)((uint32_t)e / (uint32_t)width) : (int)(e / width);
        const int64_t j = e - (int64_t)m * width;
        pr.acc_out[(int64_t)(m0 + m) * width + j] =
            __ldcg(P.sum + (int64_t)m * P.ntot + pr.noff + j) - P.qs[m];
    }
}

// Materialise the outputs of the previous stage (every projection's y and
// acc_out) and the step values of this prologue, each CTA its slice.  The
// pieces (one per previous projection, one for the step values) go to
// disjoint groups of the CTA's warps, so that their L2 round trips overlap
// (measured on B200: 4.0 us per stage one after another).
__device__ void materialise(const ChainPlanHeader *h, int kind, bool first_layer, bool final_phase,
                            const Prev &P, int mg, int m0)
{
    const int nprev = P.st ? P.st->nproj : 0;
    const bool step = final_phase || (kind == kStageQKV && !first_layer) || kind == kStageO ||
                      kind == kStageGU || kind == kStageDown;
    const int nc = nprev + (step ? 1 : 0);
    if (nc == 0)
        return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = warp % nc;                                  // this warp's piece
    const int tid = (warp / nc) * 32 + lane;                  // its index in the group
    const int nt = ((kNW - 1 - c) / nc + 1) * 32;             // threads of the group
    if (c < nprev) {
        const int q = c;
        write_slice(P.st->proj[q].y, P.st->proj[q].N, mg, m0, tid, nt,
                    [&](int m, int64_t j) { return prev_y4(P, q, m, j); });
        write_acc_slice(P, q, mg, m0, tid, nt);
    } else if (final_phase || (kind == kStageQKV && !first_layer)) {
        // h' = h1 + d
        write_slice(h->h, h->hidden, mg, m0, tid, nt, [&](int m, int64_t j) {
            return add4(ldcg4f(h->h1 + (int64_t)(m0 + m) * h->hidden + j), prev_y4(P, 0, m, j));
        });
    } else if (kind == kStageO) {
        write_slice(h->a, h->hidden, mg, m0, tid, nt, [&](int m, int64_t j) {
            return stage_x4(h, kStageO, false, P, m, m0 + m, j / 4);
        });
    } else if (kind == kStageGU) {
        write_slice(h->h1, h->hidden, mg, m0, tid, nt, [&](int m, int64_t j) {
            return stage_x4(h, kStageGU, false, P, m, m0 + m, j / 4);
        });
    } else {
        write_slice(h->act, h->inter, mg, m0, tid, nt, [&](int m, int64_t j) {
            return stage_x4(h, kStageDown, false, P, m, m0 + m, j / 4);
        });
    }
}

// Copy one stage plan (256 bytes) into shared memory: threads 0 .. 15.
__device__ __forceinline__ void copy_stage(ChainStagePlan *dst, const ChainStagePlan *src)
{
    static_assert(sizeof(ChainStagePlan) == 16 * 16, "stage plan copy");
    if (threadIdx.x < 16)
        reinterpret_cast<int4 *>(dst)[threadIdx.x] = reinterpret_cast<const int4 *>(src)[threadIdx.x];
}

__global__ void __launch_bounds__(kThreadsCh, 1) k_chain(const __grid_constant__ ChainParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const ChainPlanHeader *h = p.plan;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mg = p.mg, m0 = p.m0;

    // Layout: rings | activation rows (kChainGroup x xstride) | scales | reductions | barriers
    const int ring_bytes = kNW * kS * kSlotBytes;
    uint8_t *xbuf = smem + ring_bytes;
    float *sa_s = reinterpret_cast<float *>(xbuf + kChainGroup * p.xstride);   // [8] this stage
    int *qs_s = reinterpret_cast<int *>(sa_s + kChainGroup);                   // [8]
    float *scale_s = reinterpret_cast<float *>(qs_s + kChainGroup);            // [8] 127/amax
    // amax/127 and sum(q) of stage s's input at [s & 1] (a stage's outputs
    // are materialised after the next stage's prologue has written its own)
    float *psa2 = scale_s + kChainGroup;                                       // [2][8]
    int *pqs2 = reinterpret_cast<int *>(psa2 + 2 * kChainGroup);               // [2][8]
    float *pws_s = reinterpret_cast<float *>(pqs2 + 2 * kChainGroup);          // [2][4] wscales
    float *red_f = pws_s + 4 + 4;                                              // [kNW][8]
    int *red_i = reinterpret_cast<int *>(red_f + kNW * kChainGroup);           // [kNW][8]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(red_i + kNW * kChainGroup) + 15) & ~uintptr_t(15));
    int *abort_p = reinterpret_cast<int *>(bars + kNW * kS);
    volatile int *abort_flag = abort_p;
    const uint32_t bar_ring = smem_u32(bars);
    // The plan header and a ring of four stage plans (stages s - 1 .. s + 2
    // at stage s), so that the stage loop reads no plan field from global
    // memory (measured on B200: each such read an L2 round trip on the
    // path of the prologue and of the materialisation).
    ChainStagePlan *sring = reinterpret_cast<ChainStagePlan *>(
        (reinterpret_cast<uintptr_t>(abort_p + 1) + 63) & ~uintptr_t(63));
    ChainPlanHeader *hs = reinterpret_cast<ChainPlanHeader *>(sring + 4);
    UnitS *ucache = reinterpret_cast<UnitS *>(
        (reinterpret_cast<uintptr_t>(hs + 1) + 63) & ~uintptr_t(63));
    if (p.unit_cache)
        for (int i = threadIdx.x; i < h->n_stages; i += kThreadsCh)
            ucache[i] = unit_fields(stage_of(h, i));
    for (int i = threadIdx.x; i < (int)(sizeof(ChainPlanHeader) / 16); i += kThreadsCh)
        reinterpret_cast<int4 *>(hs)[i] = reinterpret_cast<const int4 *>(h)[i];
    for (int i = 0; i < 2 && i < h->n_stages; ++i)
        copy_stage(sring + i, stage_of(h, i));

    uint32_t *ctr = reinterpret_cast<uint32_t *>(p.ws);
    const int64_t buf_ints = (kChainGroup * h->max_ntot * 4 + 255) / 256 * 64;
    int32_t *sums = reinterpret_cast<int32_t *>(p.ws + 256);
    auto sum_buf = [&](int s) { return sums + (int64_t)(s % kChainSumBufs) * buf_ints; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNW * kS; ++i)
            mbar_init(bar_ring + 8 * i, 1);
        *abort_p = 0;
        fence_barrier_init();
    }
    // token rows at or past mg stay zero for the whole launch
    for (int i = threadIdx.x; i < kChainGroup * p.xstride / 16; i += kThreadsCh)
        reinterpret_cast<uint4 *>(xbuf)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    // ---- the code ring of this warp (lane 0 issues), primed across stages
    const uint32_t ring_w0 = smem_u32(smem) + warp * kS * kSlotBytes;
    const uint32_t ring_w = ring_w0 + lane * 16;
    const uint32_t bar_w = bar_ring + 8 * warp * kS;
    UnitIter prod, cons;
    prod.n_stages = h->n_stages;
    prod.cache = p.unit_cache ? ucache : nullptr;
    prod.enter(h, 0, warp);
    cons = prod;
    int issued = 0, consumed = 0;
    for (int s = 0; s < kS && prod.valid; ++s) {
        if (lane == 0)
            prod.issue(ring_w0 + s * kSlotBytes, bar_w + 8 * s);
        prod.next(h, warp);
        ++issued;
    }
    int cslot = 0;
    uint32_t cphase = 0;

    // ---- clear the first stage's sums, then the first barrier
    {
        const int64_t n = (int64_t)kChainGroup * h->max_ntot;
        int64_t lo, hi;
        cta_share(n, lo, hi);
        for (int64_t e = lo + threadIdx.x; e < hi; e += kThreadsCh)
            sum_buf(0)[e] = 0;
    }
    uint32_t nbar = 1;
    bool ok = grid_barrier(ctr, nbar++, p, abort_flag);

    Prev P;
    P.st = nullptr;
    P.sum = nullptr;
    P.ntot = 0;
    P.sa = psa2;
    P.qs = pqs2;
    P.ws = pws_s;

    const int n_stages = h->n_stages;
    for (int s = 0; s <= n_stages && ok; ++s) {
        const bool final_phase = s == n_stages;
        const ChainStagePlan *st = final_phase ? nullptr : sring + (s & 3);
        // (stage s - 2's slot: its last reader, stage s - 1's
        // materialisation, is behind the barrier)
        if (s + 2 < n_stages)
            copy_stage(sring + ((s + 2) & 3), stage_of(h, s + 2));
        const int kind = final_phase ? -1 : st->kind;
        const bool first_layer = s < 4;
        // The plan entries of the next stages, into this SM's L1 (the units
        // of stage s walk into stage s + 1's, the ring's producer further).
        if (threadIdx.x < 8 && s + 1 + (threadIdx.x >> 1) < n_stages)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint8_t *>(
                             stage_of(h, s + 1 + (threadIdx.x >> 1))) + 128 * (threadIdx.x & 1)));
        if (s > 0) {
            // (pws_s holds stage s - 1's wscales, loaded before the barrier)
            P.st = sring + ((s - 1) & 3);
            P.sum = sum_buf(s - 1);
            P.ntot = P.st->ntot;
            P.sa = psa2 + ((s - 1) & 1) * kChainGroup;
            P.qs = pqs2 + ((s - 1) & 1) * kChainGroup;
            P.ws = pws_s + ((s - 1) & 1) * 4;
        }

        // ---- materialise this CTA's slices of the previous stage's outputs
        // and of the step values; clear its slice of stage s + 1's sums.
        // Nothing in stage s reads them, except the down stage's input
        // (`act`): every other stage does this after its units, off the
        // critical path (measured on B200: about 2 us per stage before them).
        auto clear_next = [&]() {
            if (!final_phase && s + 1 < n_stages) {
                const int64_t n = (int64_t)kChainGroup * sring[(s + 1) & 3].ntot;
                int64_t lo, hi;
                cta_share(n, lo, hi);
                int32_t *b = sum_buf(s + 1);
                for (int64_t e = lo + threadIdx.x; e < hi; e += kThreadsCh)
                    b[e] = 0;
            }
        };
        const bool late = !final_phase && kind != kStageDown;
        if (!late) {
            materialise(hs, kind, first_layer, final_phase, P, mg, m0);
            clear_next();
        }
        if (final_phase)
            break;
        // the down stage reads SiLU(g) * u back from `act`, whole, once
        // every CTA has written its slice
        int xkind = kind;
        if (kind == kStageDown) {
            if (!grid_barrier(ctr, nbar++, p, abort_flag)) {
                ok = false;
                break;
            }
            xkind = kStageDownAct;
        }

        // ---- prologue 2: this stage's input rows, quantised into shared memory
        const int64_t K = st->K, K4 = K / 4;
        if (mg <= kRegTokens && K4 <= (int64_t)kXR * kThreadsCh) {
            // per token: the thread's elements i = tid + j * kThreadsCh, all
            // loaded at once and kept; amax over the row; 127/amax
            float4 v[kRegTokens][kXR];
            float am[kRegTokens];
#pragma unroll
            for (int m = 0; m < kRegTokens; ++m) {
                am[m] = 0.f;
                int4 ra[kXR], rb[kXR];
#pragma unroll
                for (int j = 0; j < kXR; ++j) {
                    const int64_t i = threadIdx.x + (int64_t)j * kThreadsCh;
                    ra[j] = make_int4(0, 0, 0, 0);
                    rb[j] = make_int4(0, 0, 0, 0);
                    if (m < mg && i < K4)
                        stage_raw(hs, xkind, first_layer, P, m, m0 + m, i, ra[j], rb[j]);
                }
#pragma unroll
                for (int j = 0; j < kXR; ++j) {
                    const int64_t i = threadIdx.x + (int64_t)j * kThreadsCh;
                    v[m][j] = (m < mg && i < K4) ? stage_val(xkind, first_layer, P, m, ra[j], rb[j])
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int m = 0; m < kRegTokens; ++m) {
#pragma unroll
                for (int j = 0; j < kXR; ++j)
                    am[m] = fmaxf(am[m], fmaxf(fmaxf(fabsf(v[m][j].x), fabsf(v[m][j].y)),
                                               fmaxf(fabsf(v[m][j].z), fabsf(v[m][j].w))));
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    am[m] = fmaxf(am[m], __shfl_xor_sync(0xffffffffu, am[m], o));
                if (lane == 0 && m < mg)
                    red_f[warp * kChainGroup + m] = am[m];
            }
            __syncthreads();
            // quantise the kept values into shared memory, with sum(q) per
            // token; every thread reduces the warps' maxima itself, so no
            // second barrier precedes the quantisation
#pragma unroll
            for (int m = 0; m < kRegTokens; ++m) {
                if (m >= mg)
                    break;
                float a = 0.f;
                for (int w = 0; w < kNW; ++w)
                    a = fmaxf(a, red_f[w * kChainGroup + m]);
                const float sc = a == 0.f ? 0.f : __fdiv_rn(127.f, a);
                const bool zero = sc == 0.f;
                uint32_t *row = reinterpret_cast<uint32_t *>(xbuf + m * p.xstride);
                int sq = 0;
#pragma unroll
                for (int j = 0; j < kXR; ++j) {
                    const int64_t i = threadIdx.x + (int64_t)j * kThreadsCh;
                    if (i < K4)
                        row[i] = quant4c(v[m][j], sc, zero, sq);
                }
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                if (lane == 0)
                    red_i[warp * kChainGroup + m] = sq;
            }
            __syncthreads();
            // this stage's scales serve the next prologue's rescale (read
            // after the grid barrier)
            if (threadIdx.x < mg) {
                int q = 0;
                float a = 0.f;
                for (int w = 0; w < kNW; ++w) {
                    q += red_i[w * kChainGroup + threadIdx.x];
                    a = fmaxf(a, red_f[w * kChainGroup + threadIdx.x]);
                }
                psa2[(s & 1) * kChainGroup + threadIdx.x] = __fdiv_rn(a, 127.f);
                pqs2[(s & 1) * kChainGroup + threadIdx.x] = q;
            }
        } else {
            // per token: amax over the row, then 127/amax (one token at a time
            // keeps a single running value per thread)
            for (int m = 0; m < mg; ++m) {
                float a = 0.f;
                for (int64_t i = threadIdx.x; i < K4; i += kThreadsCh) {
                    const float4 v = stage_x4(hs, xkind, first_layer, P, m, m0 + m, i);
                    a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                }
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
                if (lane == 0)
                    red_f[warp * kChainGroup + m] = a;
            }
            __syncthreads();
            if (threadIdx.x < mg) {
                float a = 0.f;
                for (int w = 0; w < kNW; ++w)
                    a = fmaxf(a, red_f[w * kChainGroup + threadIdx.x]);
                sa_s[threadIdx.x] = __fdiv_rn(a, 127.f);
                scale_s[threadIdx.x] = a == 0.f ? 0.f : __fdiv_rn(127.f, a);
            }
            __syncthreads();
            // quantise the rows into shared memory, with sum(q) per token
            for (int m = 0; m < mg; ++m) {
                const float sc = scale_s[m];
                const bool zero = sc == 0.f;
                uint32_t *row = reinterpret_cast<uint32_t *>(xbuf + m * p.xstride);
                int sq = 0;
                for (int64_t i = threadIdx.x; i < K4; i += kThreadsCh)
                    row[i] = quant4c(stage_x4(hs, xkind, first_layer, P, m, m0 + m, i), sc, zero, sq);
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                if (lane == 0)
                    red_i[warp * kChainGroup + m] = sq;
            }
            __syncthreads();
            if (threadIdx.x < mg) {
                int q = 0;
                for (int w = 0; w < kNW; ++w)
                    q += red_i[w * kChainGroup + threadIdx.x];
                qs_s[threadIdx.x] = q;
            }
            __syncthreads();
            // this stage's scales serve the next prologue's rescale
            if (threadIdx.x < mg) {
                psa2[(s & 1) * kChainGroup + threadIdx.x] = sa_s[threadIdx.x];
                pqs2[(s & 1) * kChainGroup + threadIdx.x] = qs_s[threadIdx.x];
            }
        }

        // ---- this warp's units of stage s
        const int g = lane >> 2, t = lane & 3;
        const uint32_t xrow = smem_u32(xbuf) + g * p.xstride + 16 * t;
        const uint32_t xr[1] = {xrow};
        int32_t *sb = sum_buf(s);
        const int64_t ntot = st->ntot;
        while (cons.valid && cons.s == s) {
            if (!mbar_wait(bar_w + 8 * cslot, cphase, p.ctl, abort_flag)) {
                ok = false;
                break;
            }
            int q, rbl, kt0, n;
            cons.where(q, rbl, kt0, n);
            int acc[1][4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[0][a][i] = 0;
            chunk_mma<1, kCT>(acc, ring_w + cslot * kSlotBytes, xr, (uint32_t)(kt0 * kTileK), n);
            __syncwarp();
            if (prod.valid) {
                if (lane == 0) {
                    fence_proxy_async_smem();
                    prod.issue(ring_w0 + cslot * kSlotBytes, bar_w + 8 * cslot);
                }
                prod.next(h, warp);
                ++issued;
            }
            ++consumed;
            if (++cslot == kS) {
                cslot = 0;
                cphase ^= 1u;
            }
            // partial sums of rows 16 rbl + g (+8), tokens 2t (+1)
            const int64_t N = st->proj[q].N, noff = st->proj[q].noff;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = 2 * t + (i & 1);
                const int64_t row = (int64_t)rbl * kTileRows + g + 8 * (i >> 1);
                if (tok < mg && row < N) {
                    const int D = acc[0][0][i] + (acc[0][1][i] >> 2) + (acc[0][2][i] >> 4) +
                                  (acc[0][3][i] >> 6);
                    atomicAdd(sb + tok * ntot + noff + row, D);
                }
            }
            cons.next(h, warp);
        }
        if (!ok)
            *abort_flag = 1;
        else if (late)
            clear_next();
        grid_arrive(ctr);
        if (ok && late)   // off the critical path: while the other CTAs finish
            materialise(hs, kind, first_layer, final_phase, P, mg, m0);
        // this stage's wscales for the next stage (the load's latency hides
        // in the barrier; the barrier orders the store)
        if (threadIdx.x < st->nproj)
            pws_s[(s & 1) * 4 + threadIdx.x] = __ldg(st->proj[threadIdx.x].wscale);
        ok = grid_wait(ctr, nbar++, p, abort_flag) && ok;
    }

    if (!ok) {
        // Drain: every copy this warp still has in flight lands before exit.
        WaitCtl drain = p.ctl;
        drain.timeout_ns = kDrainNsCh;
        for (int i = consumed; i < issued; ++i)
            mbar_wait(bar_w + 8 * (i % kS), (uint32_t)((i / kS) & 1), drain, nullptr);
    }
    __syncthreads();
    // The last block to finish clears the counters for the next call.
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(ctr + 1, 1u) == gridDim.x - 1) {
            ctr[0] = 0u;
            ctr[1] = 0u;
            ctr[2] = 0u;
            __threadfence();
        }
    }
}

}  // namespace

int chain_fused_smem(int64_t max_K)
{
    const int xstride = (int)(max_K + 64);
    return kNW * kS * kSlotBytes + kChainGroup * xstride + 4 * 7 * kChainGroup + 32 +
           8 * kNW * kChainGroup + 16 + 8 * kNW * kS + 64 + 4 * (int)sizeof(ChainStagePlan) +
           (int)sizeof(ChainPlanHeader) + 64;
}

cudaError_t launch_chain_fused(const ChainLaunch &L, uint32_t *err, uint64_t timeout_ns,
                               cudaStream_t stream)
{
    const ChainPlanHeader &hh = *L.host;
    const int base = chain_fused_smem(hh.max_K);
    const int cache_bytes = 64 + 64 * hh.n_stages;
    const bool cache = base + cache_bytes <= 227 * 1024;
    const int smem = base + (cache ? cache_bytes : 0);
    cudaError_t e = cudaFuncSetAttribute(k_chain, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    ChainParams p;
    memset(&p, 0, sizeof(p));
    p.plan = L.plan;
    p.ws = L.ws;
    p.xstride = (int)(hh.max_K + 64);
    p.unit_cache = cache ? 1 : 0;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    for (int64_t m0 = 0; m0 < hh.M; m0 += kChainGroup) {
        p.m0 = (int)m0;
        p.mg = (int)(hh.M - m0 < kChainGroup ? hh.M - m0 : kChainGroup);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)hh.grid);
        cfg.blockDim = dim3(kThreadsCh);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the barriers need it
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_chain, p);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace tw
