// tw_internal.h — data shared by the C-ABI layer and the kernels: the encoded
// sweep table and the launch functions of each kernel family.
#pragma once

#include <cstddef>
#include <cstdint>
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
    int64_t reserved[3];
    alignas(64) uint8_t tmap_xq[128];  // CUtensorMap of xq (prefill only)
};
static_assert(sizeof(DescRecord) == 256, "record size");

struct alignas(64) TableHeader {
    uint32_t magic;
    int32_t count;
    int64_t M;
    int64_t total_rb;
    int64_t total_tiles;
    int64_t total_ptiles;
    int64_t max_K;
    int64_t sum_K;
    int64_t reserved[1];
};
static_assert(sizeof(TableHeader) == 64, "header size");

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------ launchers
// Each returns a cudaError_t from the launch.
cudaError_t launch_ternarize(const float *W, int64_t N, int64_t K, uint8_t *packed,
                             double *mean_abs, float *wscale, void *ws, uint32_t *err,
                             cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes,
                          int32_t *invalid_count, cudaStream_t stream);
cudaError_t launch_quantize(const float *x, int64_t M, int64_t K, int8_t *xq, float *amax,
                            int32_t *qsum, cudaStream_t stream);

struct DecodeLaunch {
    const DescRecord *table;  // device records (or null: use `single`)
    int count;
    int64_t M;
    int64_t total_rb, total_tiles, max_K;
    const DescRecord *single; // host copy of a one-record sweep (table == null)
};
cudaError_t launch_decode(const DecodeLaunch &L, uint32_t *err, uint64_t timeout_ns,
                          cudaStream_t stream);

cudaError_t launch_wait_probe(uint32_t *err, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace tw
