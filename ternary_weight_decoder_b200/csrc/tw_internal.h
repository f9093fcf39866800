// tw_internal.h — data shared by the C-ABI layer and the kernels: the encoded
// sweep table and the launch functions of each kernel family.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/ternary_decoder.h"

namespace tw {

constexpr int kTileRows = 16;    // rows of W per tile (one MMA M)
constexpr int kTileK = 128;      // k per tile (the pages' 128-weight unit)
constexpr int kTileBytes = 512;  // 16 x 128 codes at 2 bits
constexpr int kDecodeMaxM = 32;  // M handled by the fused decode kernel
constexpr int64_t kDecodeMaxK = 65536;
constexpr uint32_t kTableMagic = 0x54574431u;  // "TWD1"

// One projection as the kernels see it (256 bytes, 64-byte aligned so the
// trailing TMA descriptor may be used in place from global memory).
struct alignas(64) DescRecord {
    const float *x;
    const int8_t *xq;
    const float *amax;
    const int32_t *qsum;
    const uint8_t *packed;
    const float *wscale;
    float *y;
    int32_t *acc_out;
    int64_t N, K;
    int64_t rb_begin;    // first 16-row block of this projection in the sweep
    int64_t tile_begin;  // first 16x128 code tile of this projection
    int64_t ptile_begin; // first prefill output tile of this projection
    int64_t ws_xq_off;   // decode: offset of this projection's int8 rows in ws
    int64_t cost_begin;  // decode: first cost unit of this projection (static split)
    int64_t tmap_ok;     // 1: tmap_codes holds an encoded descriptor
    alignas(64) uint8_t tmap_xq[128];     // CUtensorMap of xq (prefill only)
    alignas(64) uint8_t tmap_codes[128];  // CUtensorMap of the packed codes (prefill only)
};
static_assert(sizeof(DescRecord) == 384, "record size");

struct alignas(64) TableHeader {
    uint32_t magic;
    int32_t count;
    int64_t M;
    int64_t total_rb;
    int64_t total_units; // decode: 128-row units of the tensor-core sweep
    int64_t total_ptiles;
    int32_t max_K;       // K <= 2^24
    int32_t gemm;        // more than 32 tokens: the TW_SWEEP_GEMM_* the table was encoded for
    int64_t total_cost;  // decode: cost units of the sweep
    int64_t ws_bytes;    // decode: scratch (counter, ready flags, int8 rows, scales)
};
static_assert(sizeof(TableHeader) == 64, "header size");

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------- fused decoder-layer chain
// The plan of tw_decoder_chain_fused (host-encoded by tw_chain_plan_encode,
// copied to the device by the caller): a header, then one stage per
// (layer, {qkv, o, gate/up, down}).
constexpr uint32_t kChainPlanMagic = 0x54574332u;  // "TWC2"
constexpr int kChainGroup = 8;                     // tokens per fused launch
constexpr int kChainChunk = 6;                     // code tiles per work unit
constexpr int kChainSumBufs = 4;                   // rotating partial-sum buffers
enum ChainKind : int32_t { kStageQKV = 0, kStageO = 1, kStageGU = 2, kStageDown = 3 };

struct alignas(64) ChainProj {
    const uint8_t *packed;
    const float *wscale;
    float *y;              // [M x N] output
    int32_t *acc_out;      // [M x N] int32 output, or null
    int64_t N;
    int64_t noff;          // first column of this projection in the stage's sums
    int64_t rb_off;        // first 16-row block of this projection in the stage
    int64_t pad;
};
static_assert(sizeof(ChainProj) == 64, "chain projection");

struct alignas(64) ChainStagePlan {
    int32_t kind, nproj, K, nch;   // nch: work units (chunks) per row block
    int64_t rb_total, units, ntot; // row blocks, units (row block x chunk), sum of N
    int64_t pad[3];
    ChainProj proj[3];
};
static_assert(sizeof(ChainStagePlan) == 256, "chain stage");

struct alignas(64) ChainPlanHeader {
    uint32_t magic;
    int32_t n_stages, grid, n_layers;
    int64_t M, hidden, kv_dim, head_dim, inter;
    float *h, *v, *a, *o, *h1, *g, *u, *act, *d;
    int64_t max_ntot, max_K, chunk;
};
static_assert(sizeof(ChainPlanHeader) % 64 == 0, "chain header");

struct ChainLaunch {
    const ChainPlanHeader *plan;   // device copy
    const ChainPlanHeader *host;   // host copy (sizes)
    uint8_t *ws;
};
// Scratch of the fused chain: 256 bytes of counters (zero between calls),
// then kChainSumBufs int32 sum buffers of kChainGroup x max_ntot.
inline int64_t chain_fused_ws_bytes(const ChainPlanHeader &h)
{
    return 256 + kChainSumBufs * ((kChainGroup * h.max_ntot * 4 + 255) / 256 * 256);
}
cudaError_t launch_chain_fused(const ChainLaunch &L, uint32_t *err, uint64_t timeout_ns,
                               cudaStream_t stream);

// Element-wise steps of the decoder-layer chain (tw_chain.cu).
cudaError_t launch_gqa_expand(const float *v, float *a, int64_t M, int64_t kv_dim,
                              int64_t hidden, int64_t head_dim, cudaStream_t stream);
cudaError_t launch_add_f32(const float *x, const float *y, float *out, int64_t n,
                           cudaStream_t stream);
cudaError_t launch_silu_mul(const float *g, const float *u, float *out, int64_t n,
                            cudaStream_t stream);

// ------------------------------------------------------------ launchers
// Each returns a cudaError_t from the launch.
cudaError_t launch_ternarize(const float *W, int64_t N, int64_t K, uint8_t *packed,
                             double *mean_abs, float *wscale, void *ws, uint32_t *err,
                             cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes,
                          int32_t *invalid_count, cudaStream_t stream);
cudaError_t launch_quantize(const float *x, int64_t M, int64_t K, int8_t *xq, float *amax,
                            int32_t *qsum, cudaStream_t stream);

// Static split of a decode sweep: a 16-row block of a projection with K
// columns costs 16 units per 128-column tile plus a fixed part for its
// epilogue and loop set-up.
constexpr int64_t kRbFixedCost = 45;
__host__ __device__ inline int64_t rb_cost(int64_t K) { return 16 * (K / kTileK) + kRbFixedCost; }

struct UnitOrder;

struct DecodeLaunch {
    const DescRecord *table;  // device records (or null: use `single`)
    int count;
    int64_t M;
    int64_t total_rb, total_cost, max_K;
    const DescRecord *single; // host copy of a one-record sweep (table == null)
    uint8_t *ws;              // scratch: int8 rows at each record's ws_xq_off,
    int64_t ws_sa_off;        // then 256 bytes of amax/127, sum(q) per record
    const UnitOrder *order;   // projections by K descending (sweeps; null: single)
    int n_big;                // leading entries of `order` with K > kQuantSmallK
};
// Kernel launches one decode call makes for M tokens (quantise + groups).
int decode_launches(int64_t count, int64_t M, int64_t max_K, int n_big);
// Launches of the quantisation pass for `count` projections of M tokens.
int quant_launches(int64_t count, int64_t M, int n_big);

// Decode scratch of the single-matrix path: the M int8 rows (128-byte
// aligned), then 256 bytes: 32 floats amax/127 and 32 ints sum(q).

// Tensor-core decode sweep (tw_decode_tc.cu).  Its scratch: 256 bytes of
// counters (claim, finished blocks; zero between calls), then per projection
// its token blocks -- K/128 blocks of tc_tokens(M) rows x 128 bytes, 128-byte
// swizzled -- then per projection 256 bytes of amax/127 and sum(q).
constexpr int64_t kWsCtrBytes = 256;
// Rows of projections with K above this are quantised by 8 warps each (they
// do not fit one warp's registers); the others by as few as fill the GPU.
constexpr int64_t kQuantSmallK = 1536;
inline int tc_tokens(int64_t M) { return M <= 8 ? 8 : M <= 16 ? 16 : 32; }
// Which decode kernel runs a sweep of M tokens (measured on B200 over the
// 196 projections: the tensor-core sweep wins once the int8 MMAs of the
// register path, 4 per 8 tokens per tile, and their operand loads no longer
// keep up with HBM -- 115.7 / 117.8 us against 119.9 / 124.0 us at 12 / 16
// tokens, 83 us for the register path at 8).
#ifndef TW_TC_DECODE_MIN_M
#define TW_TC_DECODE_MIN_M 9
#endif
inline bool decode_sweep_on_tensor_cores(int64_t M) { return M >= TW_TC_DECODE_MIN_M; }
// Projections in the order their units are handed out (K descending); the
// units of entry i are [unit_begin, unit_begin + units), one per 128 rows.
struct UnitOrder {
    int32_t d;
    int32_t units;
    int64_t unit_begin;
};
static_assert(sizeof(UnitOrder) == 16, "unit order entry");
struct DecodeTcLaunch {
    const DescRecord *table;  // device records
    const UnitOrder *order;   // device copy of the order (follows the records)
    int n_big;                // leading entries of `order` with K > kQuantSmallK
    int count;
    int64_t M, total_units;
    uint8_t *ws;
    int64_t ws_sa_off;
    uint32_t *ctr;
};
cudaError_t launch_decode_tc(const DecodeTcLaunch &L, uint32_t *err, uint64_t timeout_ns,
                             cudaStream_t stream);
// Quantise every (projection, token) row into the token blocks above.
// Quantise every record's fp32 x (records without x are skipped) into its
// own xq, amax and qsum: the first launch of a sweep of more than 32 tokens
// whose descriptors give x.
cudaError_t launch_quant_own(const DescRecord *table, int count, int64_t M, cudaStream_t stream);
cudaError_t launch_quant_tc(const DescRecord *table, const UnitOrder *order, int n_big, int count,
                            int64_t M, int ntok, uint8_t *ws, int64_t ws_sa_off, cudaStream_t stream);
inline int64_t round128(int64_t b) { return (b + 127) / 128 * 128; }
cudaError_t launch_decode(const DecodeLaunch &L, uint32_t *err, uint64_t timeout_ns,
                          cudaStream_t stream);

// Weights-in-tensor-memory GEMM for more than 32 tokens (tw_mid.cu): units
// of 128 weight rows x 128 tokens, claimed from counters in 256 bytes of
// scratch (zero between calls).  Its tables carry 128-row code boxes.
struct MidLaunch {
    const DescRecord *table;  // device records
    const UnitOrder *order;   // device copy of the order (units: row tiles x token tiles)
    int count;
    int64_t M, total_units;
    uint32_t *ctr;
};
cudaError_t launch_mid(const MidLaunch &L, uint32_t *err, uint64_t timeout_ns, cudaStream_t stream);
// Work units of one projection on that path: ceil(N / 128) x ceil(M / 128).
int64_t mid_units(int64_t M, int64_t N);
// Which kernel runs a sweep of M > 32 tokens: the weights-in-TMEM GEMM up
// to TW_MID_MAX_M tokens, the expanded-weights GEMM of tw_prefill.cu above
// (measured on B200 over the 196-projection sweep: 195 / 189 / 244 / 365 us
// against 246 / 248 / 258 / 421 us at 48 / 64 / 128 / 192 tokens, 450 against
// 426 us at 256; the first streams each code byte once per 128 tokens, the
// second expands it into shared memory once per 128-row by 256-token tile).
#ifndef TW_MID_MAX_M
#define TW_MID_MAX_M 192
#endif
inline bool sweep_on_mid(int64_t M) { return M > kDecodeMaxM && M <= TW_MID_MAX_M; }
// Tokens per unit of the weights-in-TMEM GEMM (the MMA's N side): the
// narrowest of 64, 96, 128 and 192 that holds M, so that no unit is mostly
// empty (measured on B200 over the 196 projections against 128-token units
// throughout: 196.5 / 182.4 -> 159.2 / 162.4 us at 33 / 64 tokens, 188.2 /
// 191.5 -> 173.0 / 176.3 at 80 / 96, 334 / 336 / 345 -> 286 / 292 / 339 at
// 144 / 160 / 192).
inline int mid_ntok(int64_t M) { return M <= 64 ? 64 : M <= 96 ? 96 : M <= 128 ? 128 : 192; }

struct PrefillLaunch {
    const DescRecord *table;  // device records (or null: use `single`)
    int count;
    int64_t M;
    int64_t total_ptiles;
    const DescRecord *single; // host record incl. its TMA descriptor
};
cudaError_t launch_prefill(const PrefillLaunch &L, uint32_t *err, uint64_t timeout_ns,
                           cudaStream_t stream);
// Output tiles of one projection on the prefill path (128 x 256 each).
int64_t prefill_tiles(int64_t M, int64_t N);
// Encode the TMA descriptor of xq [M x K] int8 into out128 (128 bytes).
// Returns 0, -1 when the driver entry point is unavailable, or a CUresult.
int encode_xq_tmap(const int8_t *xq, int64_t M, int64_t K, int box_m, void *out128);
// Encode the TMA descriptor of the packed codes of an [N x K] matrix, seen as
// [ceil(N/16)] x [K/128] tiles of 128 32-bit words (one box = box_rb row
// blocks x box_kt consecutive k tiles; row blocks and k tiles past the
// matrix read as zero, which is the code -1 + 1 = 0 after expansion).
int encode_codes_tmap(const uint8_t *packed, int64_t N, int64_t K, int box_rb, int box_kt,
                      void *out128);
// k tiles per pipeline stage of the tensor-core decode (tw_decode_tc.cu) and
// of the weights-in-TMEM GEMM (tw_mid.cu): one barrier wait and one commit
// of the MMA thread cover that many k tiles.  Measured on B200 over the
// 196 projections: six tiles (K = 1536 is two stages) against four, the
// tensor-core decode at 9 / 16 / 24 / 32 tokens 113.3 / 117.8 / 129.6 /
// 136.3 -> 105.9 / 111.7 / 126.7 / 134.3 us; for the weights-in-TMEM GEMM
// three or four tiles were slower than two (fewer load stages fit).
#ifndef TW_TC_GROUP
#define TW_TC_GROUP 6
#endif
constexpr int kTcGroup = TW_TC_GROUP;
#ifndef TW_MID_GROUP
#define TW_MID_GROUP 2
#endif
constexpr int kMidGroup = TW_MID_GROUP;

cudaError_t launch_wait_probe(uint32_t *err, uint64_t timeout_ns, cudaStream_t stream);

// Address of the per-device error word on the current device (TW_OK or a
// TW_ERR_* status; the message is kept for tw_last_error()).
int error_word(uint32_t **out);
// Record a message for tw_last_error() and return `code`.
int record_error(int code, const char *msg);
// Clear this host thread's last-error message (every entry point does so
// first).
void clear_error();

// Device addresses of a __device__ variable, one per device, each valid
// for the context it was looked up in (re-resolved when the current
// context's id changes, as after cudaDeviceReset).
struct SymbolCache {
    static constexpr int kDevices = 64;
    std::mutex mu;
    void *addr[kDevices] = {};
    unsigned long long ctx[kDevices] = {};
};
// `symbol` is the address of the __device__ variable as host code sees it
// (a host-side stand-in); *out receives its device address on the current
// device.  `what` names it in the error message.
int symbol_address(const void *symbol, SymbolCache &cache, const char *what, void **out);

}  // namespace tw
