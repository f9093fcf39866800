// tw_api.cu — the C ABI: argument checks, status codes, the per-device error
// word, sweep-table encoding and dispatch to the kernel families.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <cuda.h>

#include "tw_device.cuh"
#include "tw_internal.h"

namespace {

__device__ uint32_t g_tw_err;  // per-device error word (EFLAG_* bits)

thread_local char t_last_error[512] = "";
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s limit of an ordinary wait

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(TW_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the calling thread's current CUDA context, or 0 when there is none
// (or the driver cannot say).  Context ids are unique for the life of the
// process, so a context created after cudaDeviceReset gets a new one.
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess && f)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess && f)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Address of g_tw_err on the current device.  Looked up once per device and
// context: a device reset (a new context) makes the lookup run again.
int err_word(uint32_t **out)
{
    static tw::SymbolCache cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= tw::SymbolCache::kDevices)
        return fail(TW_ERR_UNSUPPORTED, "device index %d out of range", dev);
    {
        std::lock_guard<std::mutex> lk(cache.mu);
        if (!cache.addr[dev]) {   // first use of this device: check what it is
            int major = 0;
            e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
            if (e != cudaSuccess)
                return cuda_fail(e, "cudaDeviceGetAttribute");
            if (major != 10)
                return fail(TW_ERR_UNSUPPORTED,
                            "device %d is sm_%d0, this library is built for sm_100a", dev, major);
        }
    }
    void *p = nullptr;
    if (int rc = tw::symbol_address(reinterpret_cast<const void *>(&g_tw_err), cache,
                                    "the error word", &p))
        return rc;
    *out = static_cast<uint32_t *>(p);
    return TW_OK;
}

int check_shape(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 1)
        return fail(TW_ERR_SHAPE, "shape M=%lld N=%lld K=%lld: all must be >= 1", (long long)M,
                    (long long)N, (long long)K);
    if (K % tw::kTileK)
        return fail(TW_ERR_SHAPE, "K=%lld is not a multiple of 128", (long long)K);
    if (N > (1 << 24) || K > (1 << 24) || M > (1 << 24))
        return fail(TW_ERR_SHAPE, "shape M=%lld N=%lld K=%lld exceeds 2^24", (long long)M,
                    (long long)N, (long long)K);
    return TW_OK;
}

size_t round256(int64_t b) { return (size_t)((b + 255) / 256 * 256); }

// One projection on the tensor-core prefill path (any M >= 1).
int run_prefill_single(const int8_t *xq, const float *amax, const int32_t *qsum, int64_t M,
                       int64_t N, int64_t K, const void *packed, const float *wscale, float *y,
                       int32_t *acc_out, uint32_t *err, cudaStream_t stream)
{
    tw::DescRecord r;
    memset(&r, 0, sizeof(r));
    r.xq = xq;
    r.amax = amax;
    r.qsum = qsum;
    r.packed = static_cast<const uint8_t *>(packed);
    r.wscale = wscale;
    r.y = y;
    r.acc_out = acc_out;
    r.N = N;
    r.K = K;
    int rc = tw::encode_xq_tmap(xq, M, K, 128, r.tmap_xq);   // the 128-token tiles of the GEMM
    if (!rc)
        rc = tw::encode_codes_tmap(r.packed, N, K, 16, 1, r.tmap_codes);
    if (rc)
        return fail(TW_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", rc);
    tw::PrefillLaunch L{};
    L.table = nullptr;
    L.single = &r;
    L.count = 1;
    L.M = M;
    L.total_ptiles = tw::prefill_tiles(M, N);
    cudaError_t e = tw::launch_prefill(L, err, kWaitNs, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "prefill launch");
}

// ------------------------------------------------ decoder-layer chain
// What one of a layer's four sweep tables must hold for the chain buffers.
struct ChainStage {
    const char *name;
    int count;
    int64_t N[3];
    int64_t K;
    const float *x;       // every projection's x
    const float *y[3];    // required y per projection (null: any)
};

// The nine chain buffers as byte ranges.
struct ChainRange {
    const char *name;
    uintptr_t lo, hi;
};

void chain_ranges(const tw_chain_buffers &b, ChainRange r[9])
{
    const int64_t f = 4 * b.M;
    const struct { const char *n; const float *p; int64_t w; } bufs[9] = {
        {"h", b.h, b.hidden}, {"v", b.v, b.kv_dim}, {"a", b.a, b.hidden},
        {"o", b.o, b.hidden}, {"h1", b.h1, b.hidden}, {"g", b.g, b.inter},
        {"u", b.u, b.inter}, {"act", b.act, b.inter}, {"d", b.d, b.hidden}};
    for (int i = 0; i < 9; ++i) {
        const uintptr_t lo = reinterpret_cast<uintptr_t>(bufs[i].p);
        r[i] = ChainRange{bufs[i].n, lo, lo + (uintptr_t)(f * bufs[i].w)};
    }
}

// Name of the first chain buffer that [lo, hi) overlaps, or null.
const char *overlaps_chain(uintptr_t lo, uintptr_t hi, const ChainRange r[9])
{
    for (int i = 0; i < 9; ++i)
        if (lo < r[i].hi && r[i].lo < hi)
            return r[i].name;
    return nullptr;
}

int check_chain_stage(const void *host, const void *dev, const ChainStage &st, int64_t M, int layer,
                      const ChainRange ranges[9])
{
    if (!host || !dev)
        return fail(TW_ERR_NULL, "chain layer %d: %s table missing", layer, st.name);
    if ((reinterpret_cast<uintptr_t>(dev) & 63u) != 0)
        return fail(TW_ERR_ALIGN, "chain layer %d: %s device table must be 64-byte aligned", layer,
                    st.name);
    const auto *hdr = static_cast<const tw::TableHeader *>(host);
    if (hdr->magic != tw::kTableMagic)
        return fail(TW_ERR_CORRUPT, "chain layer %d: %s table was not produced by "
                    "tw_sweep_table_encode", layer, st.name);
    if (hdr->count != st.count || hdr->M != M)
        return fail(TW_ERR_SHAPE, "chain layer %d: %s table has %d projections at M=%lld, "
                    "expected %d at M=%lld", layer, st.name, hdr->count, (long long)hdr->M,
                    st.count, (long long)M);
    const auto *r = reinterpret_cast<const tw::DescRecord *>(hdr + 1);
    for (int i = 0; i < st.count; ++i) {
        if (r[i].N != st.N[i] || r[i].K != st.K)
            return fail(TW_ERR_SHAPE, "chain layer %d: %s projection %d is %lldx%lld, expected "
                        "%lldx%lld", layer, st.name, i, (long long)r[i].N, (long long)r[i].K,
                        (long long)st.N[i], (long long)st.K);
        if (r[i].x != st.x)
            return fail(TW_ERR_SHAPE, "chain layer %d: %s projection %d does not read its chain "
                        "input buffer", layer, st.name, i);
        if (st.y[i] && r[i].y != st.y[i])
            return fail(TW_ERR_SHAPE, "chain layer %d: %s projection %d does not write its chain "
                        "output buffer", layer, st.name, i);
        // An output that is not the projection's own chain buffer must lie
        // outside all of them: the chain reads those while the sweep writes.
        const uintptr_t bytes = (uintptr_t)(4 * M * r[i].N);
        const uintptr_t ylo = reinterpret_cast<uintptr_t>(r[i].y);
        if (!st.y[i])
            if (const char *hit = overlaps_chain(ylo, ylo + bytes, ranges))
                return fail(TW_ERR_SHAPE, "chain layer %d: %s projection %d writes into chain "
                            "buffer %s", layer, st.name, i, hit);
        const uintptr_t alo = reinterpret_cast<uintptr_t>(r[i].acc_out);
        if (r[i].acc_out)
            if (const char *hit = overlaps_chain(alo, alo + bytes, ranges))
                return fail(TW_ERR_SHAPE, "chain layer %d: %s projection %d has its integer "
                            "outputs in chain buffer %s", layer, st.name, i, hit);
    }
    return TW_OK;
}

// The four stages of one layer for the buffers b.
void chain_stages(const tw_chain_buffers &b, ChainStage st[4])
{
    st[0] = ChainStage{"qkv", 3, {b.hidden, b.kv_dim, b.kv_dim}, b.hidden, b.h, {nullptr, nullptr, b.v}};
    st[1] = ChainStage{"o", 1, {b.hidden, 0, 0}, b.hidden, b.a, {b.o, nullptr, nullptr}};
    st[2] = ChainStage{"gate/up", 2, {b.inter, b.inter, 0}, b.hidden, b.h1, {b.g, b.u, nullptr}};
    st[3] = ChainStage{"down", 1, {b.hidden, 0, 0}, b.inter, b.act, {b.d, nullptr, nullptr}};
}

void layer_tables(const tw_chain_layer &L, const void *host[4], const void *dev[4])
{
    host[0] = L.qkv_host, dev[0] = L.qkv_dev;
    host[1] = L.o_host, dev[1] = L.o_dev;
    host[2] = L.gu_host, dev[2] = L.gu_dev;
    host[3] = L.down_host, dev[3] = L.down_dev;
}

int check_chain_buffers(const tw_chain_buffers *b)
{
    if (!b)
        return fail(TW_ERR_NULL, "tw_decoder_chain: buffers required");
    const void *ptrs[] = {b->h, b->v, b->a, b->o, b->h1, b->g, b->u, b->act, b->d};
    for (const void *q : ptrs) {
        if (!q)
            return fail(TW_ERR_NULL, "tw_decoder_chain: every chain buffer is required");
        if (!aligned16(q))
            return fail(TW_ERR_ALIGN, "tw_decoder_chain: chain buffers must be 16-byte aligned");
    }
    if (b->M < 1 || b->M > tw::kDecodeMaxM)
        return fail(TW_ERR_SHAPE, "tw_decoder_chain: M=%lld outside 1..%d (decode only)",
                    (long long)b->M, tw::kDecodeMaxM);
    if (b->hidden <= 0 || b->inter <= 0 || b->hidden % 128 || b->inter % 128)
        return fail(TW_ERR_SHAPE, "tw_decoder_chain: hidden and inter must be positive "
                    "multiples of 128");
    if (b->head_dim <= 0 || b->kv_dim <= 0 || b->hidden % b->head_dim || b->kv_dim % b->head_dim ||
        (b->hidden / b->head_dim) % (b->kv_dim / b->head_dim))
        return fail(TW_ERR_SHAPE, "tw_decoder_chain: hidden and kv_dim must be whole heads of "
                    "head_dim, the query heads an equal number per KV head");
    ChainRange r[9];
    chain_ranges(*b, r);
    for (int i = 0; i < 9; ++i)
        for (int j = i + 1; j < 9; ++j)
            if (r[i].lo < r[j].hi && r[j].lo < r[i].hi)
                return fail(TW_ERR_SHAPE, "tw_decoder_chain: chain buffers %s and %s overlap",
                            r[i].name, r[j].name);
    return TW_OK;
}

}  // namespace

namespace tw {
int error_word(uint32_t **out) { return err_word(out); }
int record_error(int code, const char *msg) { return fail(code, "%s", msg); }
void clear_error() { t_last_error[0] = 0; }

int symbol_address(const void *symbol, SymbolCache &c, const char *what, void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= SymbolCache::kDevices)
        return fail(TW_ERR_UNSUPPORTED, "device index %d out of range", dev);
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lk(c.mu);
    if (!c.addr[dev] || id == 0 || c.ctx[dev] != id) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, symbol);
        if (e != cudaSuccess || !p)
            return fail(TW_ERR_CUDA, "cudaGetSymbolAddress(%s): %s", what,
                        e != cudaSuccess ? cudaGetErrorString(e) : "null address");
        c.addr[dev] = p;
        c.ctx[dev] = id ? id : current_context_id();   // the lookup made a context current
    }
    *out = c.addr[dev];
    return TW_OK;
}
}  // namespace tw

extern "C" {

size_t tw_packed_bytes(int64_t N, int64_t K)
{
    if (N < 1 || K < 1)
        return 0;
    return (size_t)(tw::ceil_div(N, tw::kTileRows) * tw::kTileRows) * (size_t)K / 4;
}

size_t tw_ternarize_workspace_bytes(int64_t N, int64_t K)
{
    (void)K;
    if (N < 1)
        return 0;
    return (size_t)((256 + 8 * N + 255) / 256 * 256);
}

const char *tw_last_error(void) { return t_last_error; }

int tw_ternarize_pack(const float *W, int64_t N, int64_t K, void *packed, size_t packed_bytes,
                      double *mean_abs, float *wscale, void *ws, size_t ws_bytes,
                      tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!W || !packed || !wscale || !ws)
        return fail(TW_ERR_NULL, "tw_ternarize_pack: W, packed, wscale and ws are required");
    if (int rc = check_shape(1, N, K))
        return rc;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(ws) || !aligned16(wscale) ||
        (mean_abs && !aligned16(mean_abs)))
        return fail(TW_ERR_ALIGN, "tw_ternarize_pack: pointers must be 16-byte aligned");
    if (packed_bytes < tw_packed_bytes(N, K))
        return fail(TW_ERR_BUFSIZE, "packed buffer %zu < %zu bytes", packed_bytes,
                    tw_packed_bytes(N, K));
    if (ws_bytes < tw_ternarize_workspace_bytes(N, K))
        return fail(TW_ERR_BUFSIZE, "workspace %zu < %zu bytes", ws_bytes,
                    tw_ternarize_workspace_bytes(N, K));
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    cudaError_t e = tw::launch_ternarize(W, N, K, static_cast<uint8_t *>(packed), mean_abs,
                                         wscale, ws, err, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "ternarize launch");
}

int tw_unpack_codes(const void *packed, int64_t N, int64_t K, int8_t *codes,
                    int32_t *invalid_count, tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!packed || !codes)
        return fail(TW_ERR_NULL, "tw_unpack_codes: packed and codes are required");
    if (int rc = check_shape(1, N, K))
        return rc;
    if (!aligned16(packed) || !aligned16(codes) || (invalid_count && !aligned16(invalid_count)))
        return fail(TW_ERR_ALIGN, "tw_unpack_codes: pointers must be 16-byte aligned");
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    cudaError_t e = tw::launch_unpack(static_cast<const uint8_t *>(packed), N, K, codes,
                                      invalid_count, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "unpack launch");
}

int tw_quantize_act(const float *x, int64_t M, int64_t K, int8_t *xq, float *amax, int32_t *qsum,
                    tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!x || !xq || !amax)
        return fail(TW_ERR_NULL, "tw_quantize_act: x, xq and amax are required");
    if (int rc = check_shape(M, 1, K))
        return rc;
    if (!aligned16(x) || !aligned16(xq) || !aligned16(amax) || (qsum && !aligned16(qsum)))
        return fail(TW_ERR_ALIGN, "tw_quantize_act: pointers must be 16-byte aligned");
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    cudaError_t e = tw::launch_quantize(x, M, K, xq, amax, qsum, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "quantize launch");
}

size_t tw_linear_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    (void)N;
    if (M <= tw::kDecodeMaxM)
        return (size_t)(tw::round128(M * K) + 256);
    return round256(M * K) + 2 * round256(M * 4);
}

int tw_ternary_linear(const float *x, int64_t M, int64_t N, int64_t K, const void *packed,
                      const float *wscale, float *y, int32_t *acc_out, void *ws, size_t ws_bytes,
                      tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!x || !packed || !wscale || !y)
        return fail(TW_ERR_NULL, "tw_ternary_linear: x, packed, wscale and y are required");
    if (int rc = check_shape(M, N, K))
        return rc;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(wscale) || !aligned16(y) ||
        (acc_out && !aligned16(acc_out)))
        return fail(TW_ERR_ALIGN, "tw_ternary_linear: pointers must be 16-byte aligned");
    if (ws_bytes < tw_linear_workspace_bytes(M, N, K) || (ws_bytes && !ws))
        return fail(TW_ERR_BUFSIZE, "workspace %zu < %zu bytes", ws_bytes,
                    tw_linear_workspace_bytes(M, N, K));
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    if (M <= tw::kDecodeMaxM) {
        if (K > tw::kDecodeMaxK)
            return fail(TW_ERR_SHAPE, "decode path supports K <= %lld", (long long)tw::kDecodeMaxK);
        tw::DescRecord r;
        memset(&r, 0, sizeof(r));
        r.x = x;
        r.packed = static_cast<const uint8_t *>(packed);
        r.wscale = wscale;
        r.y = y;
        r.acc_out = acc_out;
        r.N = N;
        r.K = K;
        r.ws_xq_off = 0;
        tw::DecodeLaunch L{};
        L.table = nullptr;
        L.single = &r;
        L.count = 1;
        L.M = M;
        L.total_rb = tw::ceil_div(N, tw::kTileRows);
        L.total_cost = L.total_rb * tw::rb_cost(K);
        L.max_K = K;
        L.ws = static_cast<uint8_t *>(ws);
        L.ws_sa_off = tw::round128(M * K);
        cudaError_t e = tw::launch_decode(L, err, kWaitNs, stream);
        return e == cudaSuccess ? TW_OK : cuda_fail(e, "decode launch");
    }
    // Prefill: quantise into the workspace, then the tensor-core GEMM.
    int8_t *xq = static_cast<int8_t *>(ws);
    float *amax = reinterpret_cast<float *>(static_cast<char *>(ws) + round256(M * K));
    int32_t *qsum = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(amax) + round256(M * 4));
    cudaError_t e = tw::launch_quantize(x, M, K, xq, amax, qsum, stream);
    if (e != cudaSuccess)
        return cuda_fail(e, "quantize launch");
    return run_prefill_single(xq, amax, qsum, M, N, K, packed, wscale, y, acc_out, err, stream);
}

int tw_ternary_linear_q(const int8_t *xq, const float *amax, const int32_t *qsum, int64_t M,
                        int64_t N, int64_t K, const void *packed, const float *wscale, float *y,
                        int32_t *acc_out, void *ws, size_t ws_bytes, tw_stream_t stream)
{
    t_last_error[0] = 0;
    (void)ws;
    (void)ws_bytes;
    if (!xq || !amax || !qsum || !packed || !wscale || !y)
        return fail(TW_ERR_NULL,
                    "tw_ternary_linear_q: xq, amax, qsum, packed, wscale and y are required");
    if (int rc = check_shape(M, N, K))
        return rc;
    if (!aligned16(xq) || !aligned16(amax) || !aligned16(qsum) || !aligned16(packed) ||
        !aligned16(wscale) || !aligned16(y) || (acc_out && !aligned16(acc_out)))
        return fail(TW_ERR_ALIGN, "tw_ternary_linear_q: pointers must be 16-byte aligned");
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    return run_prefill_single(xq, amax, qsum, M, N, K, packed, wscale, y, acc_out, err, stream);
}

size_t tw_sweep_table_bytes(int count)
{
    if (count < 1)
        return 0;
    return sizeof(tw::TableHeader) + (size_t)count * (sizeof(tw::DescRecord) + sizeof(tw::UnitOrder));
}

int tw_sweep_table_encode(const tw_proj_desc *descs, int count, int64_t M, void *table,
                          size_t table_bytes)
{
    return tw_sweep_table_encode_gemm(descs, count, M, TW_SWEEP_GEMM_AUTO, table, table_bytes);
}

int tw_sweep_table_encode_gemm(const tw_proj_desc *descs, int count, int64_t M, int gemm,
                               void *table, size_t table_bytes)
{
    t_last_error[0] = 0;
    if (!descs || !table)
        return fail(TW_ERR_NULL, "tw_sweep_table_encode: descs and table are required");
    if (gemm != TW_SWEEP_GEMM_AUTO && gemm != TW_SWEEP_GEMM_EXPANDED)
        return fail(TW_ERR_SHAPE, "gemm=%d is not a TW_SWEEP_GEMM_* value", gemm);
    if (count < 1)
        return fail(TW_ERR_SHAPE, "count=%d must be >= 1", count);
    if (table_bytes < tw_sweep_table_bytes(count))
        return fail(TW_ERR_BUFSIZE, "table buffer %zu < %zu bytes", table_bytes,
                    tw_sweep_table_bytes(count));
    if (M < 1 || M > (1 << 24))
        return fail(TW_ERR_SHAPE, "M=%lld out of range", (long long)M);
    const bool decode = M <= tw::kDecodeMaxM;
    const bool mid = gemm == TW_SWEEP_GEMM_AUTO && tw::sweep_on_mid(M);
    auto *hdr = static_cast<tw::TableHeader *>(table);
    auto *recs = reinterpret_cast<tw::DescRecord *>(hdr + 1);
    memset(table, 0, tw_sweep_table_bytes(count));
    int64_t rb = 0, tiles = 0, ptiles = 0, max_K = 0, cost = 0;
    // decode scratch: counters | per projection its token rows or blocks
    // (room for tc_tokens(M) >= M rows of K bytes) | scales
    int64_t ws_off = tw::kWsCtrBytes;
    const int64_t rows = decode ? tw::tc_tokens(M) : 0;
    for (int d = 0; d < count; ++d) {
        const tw_proj_desc &s = descs[d];
        if (int rc = check_shape(M, s.N, s.K))
            return fail(rc, "descriptor %d: %s", d, t_last_error);
        if (decode && s.K > tw::kDecodeMaxK)
            return fail(TW_ERR_SHAPE, "descriptor %d: decode path supports K <= %lld", d,
                        (long long)tw::kDecodeMaxK);
        if (!s.packed || !s.wscale || !s.y || (decode && !s.x))
            return fail(TW_ERR_NULL, "descriptor %d: x, packed, wscale and y are required", d);
        if (!decode && (!s.xq || !s.amax || !s.qsum))
            return fail(TW_ERR_NULL, "descriptor %d: prefill needs xq, amax and qsum", d);
        if (!aligned16(s.packed) || !aligned16(s.wscale) || !aligned16(s.y) ||
            (s.x && !aligned16(s.x)) || (s.acc_out && !aligned16(s.acc_out)) ||
            (s.xq && !aligned16(s.xq)) || (s.amax && !aligned16(s.amax)) ||
            (s.qsum && !aligned16(s.qsum)))
            return fail(TW_ERR_ALIGN, "descriptor %d: pointers must be 16-byte aligned", d);
        tw::DescRecord &r = recs[d];
        r.x = s.x;
        r.xq = s.xq;
        r.amax = s.amax;
        r.qsum = s.qsum;
        r.packed = static_cast<const uint8_t *>(s.packed);
        r.wscale = s.wscale;
        r.y = s.y;
        r.acc_out = s.acc_out;
        r.N = s.N;
        r.K = s.K;
        r.rb_begin = rb;
        r.tile_begin = tiles;
        r.ptile_begin = ptiles;
        {
            // M > 32: xq tiles of 128 tokens; code boxes of 128 rows x 4 k
            // tiles (tensor-core decode), 128 rows x 2 k tiles (weights-in-TMEM
            // GEMM) or 256 rows x 1 k tile (expanded-weights GEMM).  Without a
            // CUDA driver (-1) a decode table is still encoded for its sizes;
            // the sweep refuses it.
            int rc = decode ? 0 : tw::encode_xq_tmap(s.xq, M, s.K, mid ? tw::mid_ntok(M) : 128, r.tmap_xq);
            if (!rc)
                rc = tw::encode_codes_tmap(r.packed, s.N, s.K, decode || mid ? 8 : 16,
                                           decode ? tw::kTcGroup : mid ? tw::kMidGroup : 1,
                                           r.tmap_codes);
            if (rc && !(decode && rc == -1))
                return fail(TW_ERR_CUDA, "descriptor %d: cuTensorMapEncodeTiled failed (%d)", d,
                            rc);
            r.tmap_ok = rc == 0;
        }
        ptiles += tw::prefill_tiles(M, s.N);
        const int64_t nrb = tw::ceil_div(s.N, tw::kTileRows);
        if (decode) {
            r.ws_xq_off = ws_off;
            ws_off += tw::round128(rows * s.K);
            r.cost_begin = cost;
            cost += nrb * tw::rb_cost(s.K);
        }
        rb += nrb;
        tiles += nrb * (s.K / tw::kTileK);
        max_K = s.K > max_K ? s.K : max_K;
    }
    if (rb > INT32_MAX || tiles > ((int64_t)1 << 40))
        return fail(TW_ERR_SHAPE, "sweep too large: %lld row blocks", (long long)rb);
    // Order of the tensor-core sweep's units: projections of larger K first
    // (stable), 128 rows per unit.
    auto *order = reinterpret_cast<tw::UnitOrder *>(recs + count);
    for (int d = 0; d < count; ++d)
        order[d].d = d;
    std::stable_sort(order, order + count, [&](const tw::UnitOrder &a, const tw::UnitOrder &b) {
        return recs[a.d].K > recs[b.d].K;
    });
    int64_t units = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t n = recs[order[i].d].N;
        order[i].units = (int32_t)(decode ? tw::ceil_div(n, 128) : tw::mid_units(M, n));
        order[i].unit_begin = units;
        units += order[i].units;
    }
    if (units > INT32_MAX)
        return fail(TW_ERR_SHAPE, "sweep too large: %lld units", (long long)units);
    hdr->magic = tw::kTableMagic;
    hdr->count = count;
    hdr->M = M;
    hdr->total_rb = rb;
    hdr->total_units = units;
    hdr->total_ptiles = ptiles;
    // decode: counters, rows and scales; more tokens: the unit counters of the
    // weights-in-TMEM kernel
    hdr->ws_bytes = decode ? ws_off + 256 * (int64_t)count : (mid ? tw::kWsCtrBytes : 0);
    hdr->max_K = (int32_t)max_K;
    hdr->gemm = decode ? TW_SWEEP_GEMM_AUTO : gemm;
    hdr->total_cost = cost;
    return TW_OK;
}

size_t tw_sweep_workspace_bytes(const void *table_host)
{
    const auto *hdr = static_cast<const tw::TableHeader *>(table_host);
    if (!hdr || hdr->magic != tw::kTableMagic)
        return 0;
    return (size_t)hdr->ws_bytes;
}

// Whether a sweep of more than 32 tokens quantises some descriptor's fp32 x
// itself (first launch) before the GEMM.
// Whether a host table of more than 32 tokens runs the weights-in-TMEM GEMM.
static bool table_on_mid(const tw::TableHeader *hdr)
{
    return hdr->gemm == TW_SWEEP_GEMM_AUTO && tw::sweep_on_mid(hdr->M);
}

static bool sweep_quantises_x(const tw::TableHeader *hdr)
{
    if (hdr->M <= tw::kDecodeMaxM)
        return false;
    const auto *recs = reinterpret_cast<const tw::DescRecord *>(hdr + 1);
    for (int d = 0; d < hdr->count; ++d)
        if (recs[d].x)
            return true;
    return false;
}

// Projections of a host table with K > kQuantSmallK (they lead the unit order).
static int big_k_projections(const tw::TableHeader *hdr)
{
    const auto *recs = reinterpret_cast<const tw::DescRecord *>(hdr + 1);
    int n = 0;
    for (int d = 0; d < hdr->count; ++d)
        n += recs[d].K > tw::kQuantSmallK;
    return n;
}

int tw_decoder_projection_sweep(const void *table_host, const void *table_dev, void *ws,
                                size_t ws_bytes, tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!table_host || !table_dev)
        return fail(TW_ERR_NULL, "tw_decoder_projection_sweep: host and device tables required");
    if ((reinterpret_cast<uintptr_t>(table_dev) & 63u) != 0)
        return fail(TW_ERR_ALIGN, "device table must be 64-byte aligned");
    const auto *hdr = static_cast<const tw::TableHeader *>(table_host);
    if (hdr->magic != tw::kTableMagic || hdr->count < 1)
        return fail(TW_ERR_CORRUPT, "host table was not produced by tw_sweep_table_encode");
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    if (table_on_mid(hdr)) {
        if (ws_bytes < (size_t)hdr->ws_bytes || !ws)
            return fail(TW_ERR_BUFSIZE, "sweep workspace %zu < %lld bytes", ws_bytes,
                        (long long)hdr->ws_bytes);
        if (!aligned16(ws))
            return fail(TW_ERR_ALIGN, "sweep workspace must be 16-byte aligned");
        const auto *recs_dev = reinterpret_cast<const tw::DescRecord *>(
            static_cast<const tw::TableHeader *>(table_dev) + 1);
        if (sweep_quantises_x(hdr)) {
            cudaError_t e = tw::launch_quant_own(recs_dev, hdr->count, hdr->M, stream);
            if (e != cudaSuccess)
                return cuda_fail(e, "sweep quantisation launch");
        }
        tw::MidLaunch P{};
        P.table = recs_dev;
        P.order = reinterpret_cast<const tw::UnitOrder *>(recs_dev + hdr->count);
        P.count = hdr->count;
        P.M = hdr->M;
        P.total_units = hdr->total_units;
        P.ctr = reinterpret_cast<uint32_t *>(ws);
        cudaError_t e = tw::launch_mid(P, err, kWaitNs, stream);
        return e == cudaSuccess ? TW_OK : cuda_fail(e, "prefill sweep launch");
    }
    if (hdr->M > tw::kDecodeMaxM) {
        tw::PrefillLaunch P{};
        P.table = reinterpret_cast<const tw::DescRecord *>(
            static_cast<const tw::TableHeader *>(table_dev) + 1);
        if (sweep_quantises_x(hdr)) {
            cudaError_t e = tw::launch_quant_own(P.table, hdr->count, hdr->M, stream);
            if (e != cudaSuccess)
                return cuda_fail(e, "sweep quantisation launch");
        }
        P.single = nullptr;
        P.count = hdr->count;
        P.M = hdr->M;
        P.total_ptiles = hdr->total_ptiles;
        cudaError_t e = tw::launch_prefill(P, err, kWaitNs, stream);
        return e == cudaSuccess ? TW_OK : cuda_fail(e, "prefill sweep launch");
    }
    if (ws_bytes < (size_t)hdr->ws_bytes || !ws)
        return fail(TW_ERR_BUFSIZE, "sweep workspace %zu < %lld bytes", ws_bytes,
                    (long long)hdr->ws_bytes);
    if (!aligned16(ws))
        return fail(TW_ERR_ALIGN, "sweep workspace must be 16-byte aligned");
    const auto *recs_dev = reinterpret_cast<const tw::DescRecord *>(
        static_cast<const tw::TableHeader *>(table_dev) + 1);
    const auto *order_dev = reinterpret_cast<const tw::UnitOrder *>(recs_dev + hdr->count);
    const int n_big = big_k_projections(hdr);
    if (!tw::decode_sweep_on_tensor_cores(hdr->M)) {
        tw::DecodeLaunch L{};
        L.table = recs_dev;
        L.order = order_dev;
        L.n_big = n_big;
        L.single = nullptr;
        L.count = hdr->count;
        L.M = hdr->M;
        L.total_rb = hdr->total_rb;
        L.total_cost = hdr->total_cost;
        L.max_K = hdr->max_K;
        L.ws = static_cast<uint8_t *>(ws);
        L.ws_sa_off = hdr->ws_bytes - 256 * (int64_t)hdr->count;
        cudaError_t e = tw::launch_decode(L, err, kWaitNs, stream);
        return e == cudaSuccess ? TW_OK : cuda_fail(e, "sweep launch");
    }
    if (!reinterpret_cast<const tw::DescRecord *>(hdr + 1)->tmap_ok)
        return fail(TW_ERR_CUDA, "table was encoded without the CUDA driver's TMA encoder");
    tw::DecodeTcLaunch T{};
    T.table = recs_dev;
    T.order = order_dev;
    T.n_big = n_big;
    T.count = hdr->count;
    T.M = hdr->M;
    T.total_units = hdr->total_units;
    T.ws = static_cast<uint8_t *>(ws);
    T.ws_sa_off = hdr->ws_bytes - 256 * (int64_t)hdr->count;
    T.ctr = reinterpret_cast<uint32_t *>(ws);
    cudaError_t e = tw::launch_decode_tc(T, err, kWaitNs, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "sweep launch");
}

int tw_sweep_launches(const void *table_host)
{
    const auto *hdr = static_cast<const tw::TableHeader *>(table_host);
    if (!hdr || hdr->magic != tw::kTableMagic)
        return 0;
    if (hdr->M > tw::kDecodeMaxM)
        return sweep_quantises_x(hdr) ? 2 : 1;
    const int n_big = big_k_projections(hdr);
    if (!tw::decode_sweep_on_tensor_cores(hdr->M))
        return tw::decode_launches(hdr->count, hdr->M, hdr->max_K, n_big);
    return tw::quant_launches(hdr->count, hdr->M, n_big) + 1;  // quantise + the tensor-core sweep
}

int tw_check(tw_stream_t stream)
{
    t_last_error[0] = 0;
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t v = 0;
    e = cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return cuda_fail(e, "reading the error word");
    if (!v)
        return TW_OK;
    const uint32_t zero = 0;
    e = cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess)
        return cuda_fail(e, "clearing the error word");
    if (v & tw::EFLAG_TIMEOUT)
        return fail(TW_ERR_TIMEOUT, "a device-side wait timed out (error word 0x%x)", v);
    if (v & tw::EFLAG_NONFINITE)
        return fail(TW_ERR_NONFINITE, "non-finite weight found (error word 0x%x)", v);
    return fail(TW_ERR_CORRUPT, "kernel reported a malformed descriptor (error word 0x%x)", v);
}

int tw_debug_wait_timeout(uint64_t timeout_ns, tw_stream_t stream)
{
    t_last_error[0] = 0;
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    cudaError_t e = tw::launch_wait_probe(err, timeout_ns, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "wait probe launch");
}

size_t tw_chain_workspace_bytes(const tw_chain_layer *layers, int n_layers)
{
    if (!layers || n_layers < 1)
        return 0;
    size_t need = 0;
    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        for (int s = 0; s < 4; ++s) {
            const auto *hdr = static_cast<const tw::TableHeader *>(host[s]);
            if (!hdr || hdr->magic != tw::kTableMagic)
                return 0;
            need = std::max(need, (size_t)hdr->ws_bytes);
        }
    }
    return need;
}

int tw_chain_launches(const tw_chain_layer *layers, int n_layers)
{
    if (!layers || n_layers < 1)
        return 0;
    int n = 0;
    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        for (int s = 0; s < 4; ++s) {
            const int k = host[s] ? tw_sweep_launches(host[s]) : 0;
            if (k == 0)
                return 0;
            n += k;
        }
        n += 4;  // attention stand-in, two residual adds, SiLU * up
    }
    return n;
}

size_t tw_chain_plan_bytes(int n_layers)
{
    if (n_layers < 1)
        return 0;
    return sizeof(tw::ChainPlanHeader) + (size_t)4 * n_layers * sizeof(tw::ChainStagePlan);
}

int tw_chain_plan_encode(const tw_chain_layer *layers, int n_layers, const tw_chain_buffers *buf,
                         void *plan, size_t plan_bytes)
{
    t_last_error[0] = 0;
    if (!layers || n_layers < 1 || !plan)
        return fail(TW_ERR_NULL, "tw_chain_plan_encode: layers and plan are required");
    if (plan_bytes < tw_chain_plan_bytes(n_layers))
        return fail(TW_ERR_BUFSIZE, "tw_chain_plan_encode: plan buffer %zu < %zu bytes", plan_bytes,
                    tw_chain_plan_bytes(n_layers));
    if (int rc = check_chain_buffers(buf))
        return rc;
    const tw_chain_buffers &b = *buf;
    if (b.head_dim % 4)
        return fail(TW_ERR_SHAPE, "tw_chain_plan_encode: head_dim must be a multiple of 4");
    ChainStage st[4];
    chain_stages(b, st);
    ChainRange ranges[9];
    chain_ranges(b, ranges);
    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        for (int k = 0; k < 4; ++k)
            if (int rc = check_chain_stage(host[k], dev[k], st[k], b.M, l, ranges))
                return rc;
    }
    // The grid: one CTA per SM of the current device (148 on a B200 when no
    // device can be queried).
    int dev_id = 0, sms = 148;
    if (cudaGetDevice(&dev_id) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id) != cudaSuccess)
        sms = 148;
    cudaGetLastError();
    memset(plan, 0, tw_chain_plan_bytes(n_layers));
    auto *hdr = static_cast<tw::ChainPlanHeader *>(plan);
    auto *stages = reinterpret_cast<tw::ChainStagePlan *>(hdr + 1);
    int64_t max_ntot = 0, max_K = 0;
    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        for (int k = 0; k < 4; ++k) {
            const auto *th = static_cast<const tw::TableHeader *>(host[k]);
            const auto *r = reinterpret_cast<const tw::DescRecord *>(th + 1);
            tw::ChainStagePlan &sp = stages[4 * l + k];
            sp.kind = k;
            sp.nproj = th->count;
            sp.K = (int32_t)r[0].K;
            sp.nch = (int32_t)tw::ceil_div(r[0].K / tw::kTileK, tw::kChainChunk);
            int64_t rb = 0, ntot = 0;
            for (int i = 0; i < th->count; ++i) {
                tw::ChainProj &pr = sp.proj[i];
                pr.packed = r[i].packed;
                pr.wscale = r[i].wscale;
                pr.y = r[i].y;
                pr.acc_out = r[i].acc_out;
                pr.N = r[i].N;
                pr.noff = ntot;
                pr.rb_off = rb;
                ntot += r[i].N;
                rb += tw::ceil_div(r[i].N, tw::kTileRows);
            }
            sp.rb_total = rb;
            sp.units = rb * sp.nch;
            sp.ntot = ntot;
            if (sp.units > INT32_MAX / 2)
                return fail(TW_ERR_SHAPE, "tw_chain_plan_encode: stage too large");
            max_ntot = std::max(max_ntot, ntot);
            max_K = std::max(max_K, (int64_t)sp.K);
        }
    }
    hdr->magic = tw::kChainPlanMagic;
    hdr->n_stages = 4 * n_layers;
    hdr->grid = sms;
    hdr->n_layers = n_layers;
    hdr->M = b.M;
    hdr->hidden = b.hidden;
    hdr->kv_dim = b.kv_dim;
    hdr->head_dim = b.head_dim;
    hdr->inter = b.inter;
    hdr->h = b.h;
    hdr->v = b.v;
    hdr->a = b.a;
    hdr->o = b.o;
    hdr->h1 = b.h1;
    hdr->g = b.g;
    hdr->u = b.u;
    hdr->act = b.act;
    hdr->d = b.d;
    hdr->max_ntot = max_ntot;
    hdr->max_K = max_K;
    hdr->chunk = tw::kChainChunk;
    return TW_OK;
}

size_t tw_chain_fused_workspace_bytes(const void *plan_host)
{
    const auto *h = static_cast<const tw::ChainPlanHeader *>(plan_host);
    if (!h || h->magic != tw::kChainPlanMagic)
        return 0;
    return (size_t)tw::chain_fused_ws_bytes(*h);
}

int tw_chain_fused_launches(const void *plan_host)
{
    const auto *h = static_cast<const tw::ChainPlanHeader *>(plan_host);
    if (!h || h->magic != tw::kChainPlanMagic)
        return 0;
    return (int)tw::ceil_div(h->M, tw::kChainGroup);
}

int tw_decoder_chain_fused(const void *plan_host, const void *plan_dev, void *ws, size_t ws_bytes,
                           tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!plan_host || !plan_dev || !ws)
        return fail(TW_ERR_NULL, "tw_decoder_chain_fused: host plan, device plan and ws required");
    const auto *h = static_cast<const tw::ChainPlanHeader *>(plan_host);
    if (h->magic != tw::kChainPlanMagic || h->n_stages < 4 || h->chunk != tw::kChainChunk)
        return fail(TW_ERR_CORRUPT, "tw_decoder_chain_fused: plan was not produced by "
                    "tw_chain_plan_encode");
    if ((reinterpret_cast<uintptr_t>(plan_dev) & 63u) || !aligned16(ws))
        return fail(TW_ERR_ALIGN, "tw_decoder_chain_fused: device plan 64-byte and ws 16-byte "
                    "alignment required");
    if (ws_bytes < tw_chain_fused_workspace_bytes(plan_host))
        return fail(TW_ERR_BUFSIZE, "tw_decoder_chain_fused: workspace %zu < %zu bytes", ws_bytes,
                    tw_chain_fused_workspace_bytes(plan_host));
    uint32_t *err = nullptr;
    if (int rc = err_word(&err))
        return rc;
    int dev_id = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev_id);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id);
    if (e != cudaSuccess)
        return cuda_fail(e, "device query");
    if (sms < h->grid)
        return fail(TW_ERR_UNSUPPORTED, "tw_decoder_chain_fused: plan encoded for %d SMs, device "
                    "has %d", h->grid, sms);
    tw::ChainLaunch L{static_cast<const tw::ChainPlanHeader *>(plan_dev), h,
                      static_cast<uint8_t *>(ws)};
    e = tw::launch_chain_fused(L, err, kWaitNs, stream);
    return e == cudaSuccess ? TW_OK : cuda_fail(e, "fused chain launch");
}

int tw_decoder_chain(const tw_chain_layer *layers, int n_layers, const tw_chain_buffers *buf,
                     void *ws, size_t ws_bytes, tw_stream_t stream)
{
    t_last_error[0] = 0;
    if (!layers || n_layers < 1)
        return fail(TW_ERR_NULL, "tw_decoder_chain: at least one layer required");
    if (int rc = check_chain_buffers(buf))
        return rc;
    const tw_chain_buffers &b = *buf;
    ChainStage st[4];
    chain_stages(b, st);
    ChainRange ranges[9];
    chain_ranges(b, ranges);
    // Every table is checked before anything is launched.
    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        for (int s = 0; s < 4; ++s)
            if (int rc = check_chain_stage(host[s], dev[s], st[s], b.M, l, ranges))
                return rc;
    }
    const size_t need = tw_chain_workspace_bytes(layers, n_layers);
    if (!ws || ws_bytes < need)
        return fail(TW_ERR_BUFSIZE, "tw_decoder_chain: workspace %zu < %zu bytes", ws_bytes, need);
    if (!aligned16(ws))
        return fail(TW_ERR_ALIGN, "tw_decoder_chain: workspace must be 16-byte aligned");

    for (int l = 0; l < n_layers; ++l) {
        const void *host[4], *dev[4];
        layer_tables(layers[l], host, dev);
        int rc = tw_decoder_projection_sweep(host[0], dev[0], ws, ws_bytes, stream);
        if (rc)
            return rc;
        cudaError_t e = tw::launch_gqa_expand(b.v, b.a, b.M, b.kv_dim, b.hidden, b.head_dim, stream);
        if (e != cudaSuccess)
            return cuda_fail(e, "chain attention launch");
        if ((rc = tw_decoder_projection_sweep(host[1], dev[1], ws, ws_bytes, stream)))
            return rc;
        if ((e = tw::launch_add_f32(b.h, b.o, b.h1, b.M * b.hidden, stream)) != cudaSuccess)
            return cuda_fail(e, "chain residual launch");
        if ((rc = tw_decoder_projection_sweep(host[2], dev[2], ws, ws_bytes, stream)))
            return rc;
        if ((e = tw::launch_silu_mul(b.g, b.u, b.act, b.M * b.inter, stream)) != cudaSuccess)
            return cuda_fail(e, "chain SiLU launch");
        if ((rc = tw_decoder_projection_sweep(host[3], dev[3], ws, ws_bytes, stream)))
            return rc;
        if ((e = tw::launch_add_f32(b.h1, b.d, b.h, b.M * b.hidden, stream)) != cudaSuccess)
            return cuda_fail(e, "chain residual launch");
    }
    return TW_OK;
}

}  // extern "C"
