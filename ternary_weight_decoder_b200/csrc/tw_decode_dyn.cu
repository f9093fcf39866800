// tw_decode_dyn.cu — single-launch decode sweep for up to 4 tokens with
// dynamic load balancing (the path the 196-projection decode step takes).
//
// What it computes is the same as tw_decode.cu: per projection, q = absmax
// int8 quantisation of each token row of x, acc = q * codes^T exactly in
// integers, y = ((float)acc * (amax/127)) * mean|W| ("VibeVoice-ASR-BitNet-
// ONNX" model page, Quantization table: per-tensor ternary weights with
// s = 1/mean|W|).  Only the schedule differs.
//
// One CTA per SM, 16 warps:
//   * Quantisation, inside the launch: every (projection, token) row is
//     quantised once, by one warp of one CTA (rows dealt round-robin over
//     CTAs and warps), into int8 scratch with amax/127 and sum(q); a per-row
//     ready flag in scratch is then released.
//   * Warp 0 (producer) walks units of work — about 64 KB of packed codes
//     of one projection: first an even, contiguous share of the first 80% of
//     the units (few changes of projection), then units claimed one at a
//     time from a counter in scratch, so fast and slow SMs finish together.  For each unit it prefetches the next unit into L2,
//     brings the projection's int8 rows into one of two shared buffers once
//     their flags are set, and streams the unit's code chunks (up to 8
//     16x128 tiles, 4 KB) into a shared ring with 1-D bulk copies, writing
//     a small descriptor per slot.
//   * Warps 1..15 (consumers) take ring slots round-robin: load the chunk's
//     lane slots into registers, hand the slot back, decode the codes with
//     one AND per register into m16n8k32 u8 x s8 MMAs (one accumulator per
//     2-bit position s, scaled by 4^s), and add the partial sums of their
//     16 rows into a shared int32 accumulator of the row block.  The warp
//     that adds the last chunk of a row block writes y (and acc) for it.
//   * The last CTA to finish clears the claim counter and the row flags,
//     leaving the scratch ready for the next call.  The scratch must be
//     zero-filled before its first use.
// Every wait is bounded; a timeout sets the device error word and the block
// stops, drains its copies and exits.
#include <cstring>

#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kNC = 15;                      // consumer warps
constexpr int kThreads = (kNC + 1) * 32;
constexpr int kCT = 8;                       // max tiles per chunk
constexpr int kChunk = kCT * kTileBytes;     // 4 KB
constexpr int kXB = 2;                       // activation buffers
constexpr int kSmemLimit = 227 * 1024;
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr int kDynStaticPct = 80;            // share of units split statically
constexpr bool kDynEnabled = false;          // the sweep uses tw_decode.cu until this path is faster

// Per ring slot, written by the producer before the slot's barrier completes.
struct __align__(16) SlotDesc {
    float *y;
    int32_t *acc_out;
    int32_t N, rl;      // rows of the projection; row block within it
    float wscale;
    int16_t kt0;        // first k tile of the chunk
    uint8_t n;          // tiles in the chunk (0 = stop)
    uint8_t b;          // activation buffer
    uint8_t xpar;       // phase parity of that buffer's load
    uint8_t nch;        // chunks of this row block
    uint16_t rbslot;    // shared accumulator slot
};

struct DynParams {
    const DescRecord *table;
    int count;
    int M;
    int xs;             // activation row stride in shared memory
    int R;              // ring slots (multiple of kNC)
    int RS;             // row-block accumulator slots
    int64_t total_units;
    int64_t static_units; // units [0, static_units) are split evenly over the CTAs
    uint8_t *ws;
    int64_t flags_off;  // per-row ready flags (u32)
    int64_t sa_off;     // per-projection amax/127, sum(q) (256 B each)
    WaitCtl ctl;
};

struct Smem {
    uint32_t ring, zero, xbase, info, desc, rbacc, rbcnt, rbdone, rbuse, xrel, bars, misc;
    int xbuf_bytes;
};

__device__ __forceinline__ Smem layout(const DynParams &p, uint32_t base)
{
    Smem L;
    L.ring = base;
    L.zero = base + p.R * kChunk + 64;             // 64 mod 128
    L.xbase = L.zero + p.xs;                       // 0 mod 128 (xs = K + 64)
    L.xbuf_bytes = p.M * p.xs;
    uint32_t o = L.xbase + kXB * L.xbuf_bytes;
    o = (o + 127u) & ~127u;
    L.info = o;                 o += 256 * kXB;
    L.desc = o;                 o += sizeof(SlotDesc) * p.R;
    L.rbacc = o;                o += 4 * 16 * p.M * p.RS;
    L.rbcnt = o;                o += 4 * p.RS;
    L.rbdone = o;               o += 4 * p.RS;
    L.rbuse = o;                o += 4 * p.RS;
    L.xrel = o;                 o += 4 * kXB;
    o = (o + 15u) & ~15u;
    L.bars = o;                 o += 8 * (2 * p.R + kXB);
    L.misc = o;
    return L;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_s32(uint32_t a, int v)
{
    asm volatile("red.shared.add.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_shared(uint32_t a, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
    return old;
}

// Spin (bounded) until the shared word at a equals v.
__device__ __forceinline__ bool wait_shared_eq(uint32_t a, uint32_t v, const WaitCtl &ctl,
                                               volatile int *abort_flag)
{
    if (lds32(a) == v)
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (lds32(a) == v)
            return true;
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > ctl.timeout_ns) {
            atomicOr(ctl.err, EFLAG_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
        __nanosleep(32);
    }
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

// One warp quantises token row m of projection d (amax = max|x|,
// scale = 127/amax in IEEE fp32, q = clamp(rint(x*scale), -128, 127)).
__device__ void quantise_row(const DynParams &p, int d, int m, int lane)
{
    const DescRecord &r = p.table[d];
    const int64_t K4 = r.K / 4;
    const float4 *row = reinterpret_cast<const float4 *>(r.x + (int64_t)m * r.K);
    float a = 0.f;
#pragma unroll 8
    for (int64_t i = lane; i < K4; i += 32) {
        const float4 v = __ldg(row + i);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const bool zero = (a == 0.f);
    const float scale = zero ? 0.f : __fdiv_rn(127.f, a);
    uint32_t *dst = reinterpret_cast<uint32_t *>(p.ws + r.ws_xq_off + (int64_t)m * r.K);
    int sum = 0;
#pragma unroll 8
    for (int64_t i = lane; i < K4; i += 32)
        dst[i] = quant4(__ldg(row + i), scale, zero, sum);
#pragma unroll
    for (int o = 16; o; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        uint8_t *info = p.ws + p.sa_off + 256 * (int64_t)d;
        reinterpret_cast<float *>(info)[m] = __fdiv_rn(a, 127.f);
        reinterpret_cast<int *>(info + 128)[m] = sum;
    }
    __threadfence();
    __syncwarp();
    if (lane == 0)
        st_release_u32(reinterpret_cast<uint32_t *>(p.ws + p.flags_off) + d * p.M + m, 1u);
}

// D(16x8, s32) += A(16x32, u8, row) * B(32x8, s8, col).
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t comp(const uint4 &v, int s)
{
    return s == 0 ? v.x : s == 1 ? v.y : s == 2 ? v.z : v.w;
}

// Unit u of the sweep -> projection (scanning forward from d) and row blocks.
struct UnitPos {
    int d;
    int rb_lo, rb_hi;
};

__device__ __forceinline__ void locate_unit(const DynParams &p, int64_t u, UnitPos &up)
{
    for (;;) {
        const DescRecord &r = p.table[up.d];
        const int64_t nrb = (r.N + kTileRows - 1) / kTileRows;
        const int64_t urb = r.urb;
        const int64_t units = (nrb + urb - 1) / urb;
        if (u < r.unit_begin + units || up.d + 1 >= p.count) {
            const int64_t lo = (u - r.unit_begin) * urb;
            up.rb_lo = (int)lo;
            up.rb_hi = (int)min(nrb, lo + urb);
            return;
        }
        ++up.d;
    }
}

__global__ void __launch_bounds__(kThreads, 1) k_decode_dyn(const __grid_constant__ DynParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const Smem L = layout(p, base);
    uint8_t *const gbase = smem_raw + (base - raw);
    auto gen = [&](uint32_t s) { return gbase + (s - base); };
    SlotDesc *desc = reinterpret_cast<SlotDesc *>(gen(L.desc));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gen(L.misc));
    int *last_flag = reinterpret_cast<int *>(gen(L.misc + 4));
    const uint32_t bar_full = L.bars, bar_empty = L.bars + 8 * p.R, bar_x = L.bars + 16 * p.R;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t *ctr = reinterpret_cast<uint32_t *>(p.ws);

    // ---- set-up: barriers, counters, zero row, accumulators
    if (threadIdx.x == 0) {
        for (int i = 0; i < p.R; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, 32);
        }
        for (int b = 0; b < kXB; ++b)
            mbar_init(bar_x + 8 * b, 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < p.xs / 4; i += kThreads)
        sts32(L.zero + 4 * i, 0u);
    for (int i = threadIdx.x; i < 16 * p.M * p.RS; i += kThreads)
        sts32(L.rbacc + 4 * i, 0u);
    for (int i = threadIdx.x; i < 3 * p.RS + kXB; i += kThreads)
        sts32(L.rbcnt + 4 * i, 0u);   // rbcnt, rbdone, rbuse, xrel are contiguous
    __syncthreads();

    if (warp == 0) {
        // ============================================ producer (lane 0)
        if (lane == 0) {
            uint32_t refs[kXB] = {0, 0};
            uint32_t xloads[kXB] = {0, 0};
            int cur_d = -1, cur_b = kXB - 1;
            uint32_t chunk_seq = 0, rbseq = 0;
            bool ok = true;
            UnitPos up{0, 0, 0}, upn{0, 0, 0};
            // projection fields for the current unit
            float *y = nullptr;
            int32_t *acc_out = nullptr;
            const uint8_t *packed = nullptr;
            int32_t N = 0, KT = 0;
            float wscale = 0.f;
            // Work order: this CTA's contiguous share of the first
            // static_units units, then units claimed from the shared counter.
            int64_t su = p.static_units * blockIdx.x / gridDim.x;
            const int64_t su_end = p.static_units * (blockIdx.x + 1) / gridDim.x;
            auto next_unit = [&]() -> int64_t {
                if (su < su_end)
                    return su++;
                return p.static_units + (int64_t)atomicAdd(ctr, 1u);
            };
            int64_t u = next_unit();
            int64_t u1 = next_unit();
            if (u < p.total_units)
                locate_unit(p, u, up);
            while (u < p.total_units && ok && !*abort_flag) {
                const int64_t u2 = u1 < p.total_units ? next_unit() : p.total_units;
                // prefetch the next unit's codes into L2
                if (u1 < p.total_units) {
                    upn.d = up.d;
                    locate_unit(p, u1, upn);
                    const DescRecord &rn = p.table[upn.d];
                    const int64_t rbb = 4 * rn.K;
                    bulk_prefetch_l2(rn.packed + upn.rb_lo * rbb,
                                     (uint32_t)((upn.rb_hi - upn.rb_lo) * rbb));
                }
                if (up.d != cur_d) {
                    // new projection: its int8 rows into the next buffer
                    const int b = (cur_b + 1) % kXB;
                    if (!wait_shared_eq(L.xrel + 4 * b, refs[b], p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const DescRecord &r = p.table[up.d];
                    const uint32_t *flags =
                        reinterpret_cast<const uint32_t *>(p.ws + p.flags_off) + up.d * p.M;
                    for (int m = 0; m < p.M && ok; ++m) {
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_u32(flags + m) == 0u) {
                            if (*abort_flag || globaltimer_ns() - t0 > p.ctl.timeout_ns) {
                                if (!*abort_flag)
                                    atomicOr(p.ctl.err, EFLAG_TIMEOUT);
                                *abort_flag = 1;
                                ok = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    if (!ok)
                        break;
                    fence_proxy_async_global();
                    const uint32_t bx = bar_x + 8 * b;
                    mbar_arrive_expect_tx(bx, (uint32_t)(p.M * r.K + 256));
                    for (int m = 0; m < p.M; ++m)
                        bulk_g2s(L.xbase + b * L.xbuf_bytes + m * p.xs,
                                 p.ws + r.ws_xq_off + (int64_t)m * r.K, (uint32_t)r.K, bx);
                    bulk_g2s(L.info + 256 * b, p.ws + p.sa_off + 256 * (int64_t)up.d, 256, bx);
                    ++xloads[b];
                    refs[b] = 0;
                    sts32(L.xrel + 4 * b, 0u);
                    cur_d = up.d;
                    cur_b = b;
                    y = r.y;
                    acc_out = r.acc_out;
                    packed = r.packed;
                    N = (int32_t)r.N;
                    KT = (int32_t)(r.K / kTileK);
                    wscale = __ldg(r.wscale);
                }
                const int nch = (KT + kCT - 1) / kCT;
                for (int rb = up.rb_lo; rb < up.rb_hi && ok; ++rb) {
                    const int k = (int)(rbseq % p.RS);
                    if (rbseq >= (uint32_t)p.RS &&
                        !wait_shared_eq(L.rbdone + 4 * k, lds32(L.rbuse + 4 * k), p.ctl,
                                        abort_flag)) {
                        ok = false;
                        break;
                    }
                    sts32(L.rbuse + 4 * k, lds32(L.rbuse + 4 * k) + 1u);
                    ++rbseq;
                    for (int c = 0; c < nch; ++c) {
                        const int s = (int)(chunk_seq % p.R);
                        if (chunk_seq >= (uint32_t)p.R &&
                            !mbar_wait(bar_empty + 8 * s, ((chunk_seq / p.R) - 1) & 1, p.ctl,
                                       abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int kt0 = KT * c / nch, kt1 = KT * (c + 1) / nch;
                        SlotDesc &ds = desc[s];
                        ds.y = y;
                        ds.acc_out = acc_out;
                        ds.N = N;
                        ds.rl = rb;
                        ds.wscale = wscale;
                        ds.kt0 = (int16_t)kt0;
                        ds.n = (uint8_t)(kt1 - kt0);
                        ds.b = (uint8_t)cur_b;
                        ds.xpar = (uint8_t)((xloads[cur_b] - 1) & 1);
                        ds.nch = (uint8_t)nch;
                        ds.rbslot = (uint16_t)k;
                        const uint32_t bytes = (uint32_t)((kt1 - kt0) * kTileBytes);
                        mbar_arrive_expect_tx(bar_full + 8 * s, bytes);
                        bulk_g2s(L.ring + s * kChunk,
                                 packed + ((int64_t)rb * KT + kt0) * kTileBytes, bytes,
                                 bar_full + 8 * s);
                        ++refs[cur_b];
                        ++chunk_seq;
                    }
                }
                u = u1;
                u1 = u2;
                if (u < p.total_units)
                    locate_unit(p, u, up);
            }
            // stop: one empty descriptor for each consumer's next slot
            for (int w = 0; w < kNC; ++w) {
                const int s = (int)(chunk_seq % p.R);
                if (chunk_seq >= (uint32_t)p.R)
                    mbar_wait(bar_empty + 8 * s, ((chunk_seq / p.R) - 1) & 1, p.ctl, abort_flag);
                desc[s].n = 0;
                mbar_arrive(bar_full + 8 * s);
                ++chunk_seq;
            }
            // Drain the copies still in flight (consumers may have stopped
            // early on an abort): the last R slots and both buffers.
            WaitCtl drain = p.ctl;
            drain.timeout_ns = kDrainNs;
            const uint32_t first = chunk_seq > (uint32_t)p.R ? chunk_seq - p.R : 0u;
            for (uint32_t c = first; c < chunk_seq; ++c)
                mbar_wait(bar_full + 8 * (c % p.R), (c / p.R) & 1, drain, nullptr);
            for (int b = 0; b < kXB; ++b)
                if (xloads[b])
                    mbar_wait(bar_x + 8 * b, (xloads[b] - 1) & 1, drain, nullptr);
        }
        __syncwarp();
    } else {
        // ============================================ consumers
        const int cw = warp - 1;
        // quantise this CTA's share of the (projection, token) rows
        {
            const int64_t rows = (int64_t)p.count * p.M;
            for (int64_t r = blockIdx.x + (int64_t)gridDim.x * cw; r < rows;
                 r += (int64_t)gridDim.x * kNC)
                quantise_row(p, (int)(r / p.M), (int)(r % p.M), lane);
        }
        const int g = lane >> 2, t = lane & 3;
        bool ok = true;
        for (uint32_t c = cw;; c += kNC) {
            const int s = (int)(c % p.R);
            if (!mbar_wait(bar_full + 8 * s, (c / p.R) & 1, p.ctl, abort_flag)) {
                ok = false;
                break;
            }
            const SlotDesc ds = desc[s];
            if (ds.n == 0)
                break;
            if (!mbar_wait(bar_x + 8 * ds.b, ds.xpar, p.ctl, abort_flag)) {
                ok = false;
                break;
            }
            // all eight lane slots to registers (slots past n hold stale
            // bytes and are not used), then the slot goes back
            uint4 a[kCT];
#pragma unroll
            for (int i = 0; i < kCT; ++i)
                a[i] = lds128(L.ring + s * kChunk + i * kTileBytes + lane * 16);
            {
                uint32_t dep = 0;
#pragma unroll
                for (int i = 0; i < kCT; ++i)
                    dep ^= a[i].x ^ a[i].y ^ a[i].z ^ a[i].w;
                asm volatile("" ::"r"(dep));   // the loads have completed
            }
            mbar_arrive(bar_empty + 8 * s);

            // token rows of this lane (g < M) or the zero row
            const uint32_t xrow = (g < p.M ? L.xbase + ds.b * L.xbuf_bytes + g * p.xs : L.zero) +
                                  16 * t + (uint32_t)ds.kt0 * kTileK;
            int acc[4][4];
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[s2][i] = 0;
#pragma unroll
            for (int i = 0; i < kCT; ++i) {
                if (i < ds.n) {
                    const uint4 b0 = lds128(xrow + i * kTileK);
                    const uint4 b1 = lds128(xrow + i * kTileK + 64);
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) {
                        const uint32_t mk = 0x03030303u << (2 * s2);
                        mma_u8s8(acc[s2], a[i].x & mk, a[i].y & mk, a[i].z & mk, a[i].w & mk,
                                 comp(b0, s2), comp(b1, s2));
                    }
                }
            }
            // partial sums of rows g, g+8 for tokens 2t, 2t+1 -> shared
            const uint32_t acc_base = L.rbacc + 4 * 16 * p.M * ds.rbslot;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = 2 * t + (i & 1);
                if (tok < p.M) {
                    const int v = acc[0][i] + (acc[1][i] >> 2) + (acc[2][i] >> 4) + (acc[3][i] >> 6);
                    const int row = g + 8 * (i >> 1);
                    red_add_s32(acc_base + 4 * (row * p.M + tok), v);
                }
            }
            __threadfence_block();
            __syncwarp();
            uint32_t last = 0;
            if (lane == 0)
                last = (atom_add_shared(L.rbcnt + 4 * ds.rbslot, 1u) == (uint32_t)ds.nch - 1u);
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence_block();
                const float *sa = reinterpret_cast<const float *>(gen(L.info + 256 * ds.b));
                const int *qs = reinterpret_cast<const int *>(gen(L.info + 256 * ds.b + 128));
                for (int idx = lane; idx < 16 * p.M; idx += 32) {
                    const int row = idx / p.M, tok = idx % p.M;
                    const int64_t n = (int64_t)ds.rl * kTileRows + row;
                    const int v = (int)lds32(acc_base + 4 * idx) - qs[tok];
                    sts32(acc_base + 4 * idx, 0u);
                    if (n < ds.N) {
                        const int64_t o = (int64_t)tok * ds.N + n;
                        ds.y[o] = __fmul_rn(__fmul_rn((float)v, sa[tok]), ds.wscale);
                        if (ds.acc_out)
                            ds.acc_out[o] = v;
                    }
                }
                __syncwarp();
                if (lane == 0) {
                    sts32(L.rbcnt + 4 * ds.rbslot, 0u);
                    __threadfence_block();
                    atom_add_shared(L.rbdone + 4 * ds.rbslot, 1u);
                }
            }
            if (lane == 0)
                atom_add_shared(L.xrel + 4 * ds.b, 1u);
        }
        (void)ok;
    }

    // ---- leave the scratch ready for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(ctr + 1, 1u) == gridDim.x - 1)
            *last_flag = 1;
    }
    __syncthreads();
    if (*last_flag) {
        __threadfence();
        uint32_t *flags = reinterpret_cast<uint32_t *>(p.ws + p.flags_off);
        for (int i = threadIdx.x; i < p.count * p.M; i += kThreads)
            flags[i] = 0u;
        __syncthreads();
        if (threadIdx.x == 0) {
            ctr[0] = 0u;
            ctr[1] = 0u;
            __threadfence();
        }
    }
}

int64_t dyn_smem(int R, int RS, int M, int64_t max_K)
{
    const int64_t xs = max_K + 64;
    return 1024 + (int64_t)R * kChunk + 64 + xs + (int64_t)kXB * M * xs + 128 + 256 * kXB +
           (int64_t)sizeof(SlotDesc) * R + 4LL * 16 * M * RS + 12LL * RS + 4 * kXB + 16 +
           8LL * (2 * R + kXB) + 64;
}

}  // namespace

bool decode_dyn_supported(int64_t M, int64_t max_K)
{
    return kDynEnabled && M >= 1 && M <= kDynMaxM &&
           dyn_smem(2 * kNC, 32, (int)M, max_K) <= kSmemLimit;
}

cudaError_t launch_decode_dyn(const DecodeDynLaunch &L, uint32_t *err, uint64_t timeout_ns,
                              cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    DynParams p;
    memset(&p, 0, sizeof(p));
    p.table = L.table;
    p.count = L.count;
    p.M = (int)L.M;
    p.xs = (int)(L.max_K + 64);
    p.total_units = L.total_units;
    p.static_units = L.total_units * kDynStaticPct / 100;
    p.ws = L.ws;
    p.flags_off = L.flags_off;
    p.sa_off = L.sa_off;
    p.ctl.err = err;
    p.ctl.timeout_ns = timeout_ns;
    // deepest ring (3 or 2 slots per consumer warp), then most accumulators
    p.R = 0;
    for (int k = 3; k >= 2 && !p.R; --k)
        for (int rs = 64; rs >= 32 && !p.R; rs -= 16)
            if (dyn_smem(k * kNC, rs, p.M, L.max_K) <= kSmemLimit) {
                p.R = k * kNC;
                p.RS = rs;
            }
    if (!p.R)
        return cudaErrorInvalidValue;
    const int smem = (int)dyn_smem(p.R, p.RS, p.M, L.max_K);
    e = cudaFuncSetAttribute(k_decode_dyn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    // Cooperative launch: CTAs wait on rows other CTAs quantise, so all of
    // them must be resident at once (the launch fails rather than hangs).
    void *args[] = {(void *)&p};
    return cudaLaunchCooperativeKernel((const void *)k_decode_dyn, dim3(sms), dim3(kThreads), args,
                                       (size_t)smem, stream);
}

}  // namespace tw
