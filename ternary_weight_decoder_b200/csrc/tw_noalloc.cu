// tw_noalloc.cu — tw_ternarize_pack_noalloc: ternarise-and-pack without any
// caller-provided or library-allocated scratch.
//
// Some callers cannot allocate device memory at the point where they need a
// matrix packed: a plugin running inside a host framework that owns the whole
// device-memory budget and hands its plugins no allocator, or a loop whose
// timing rules forbid cudaMalloc (it may synchronise the device).  For them
// this entry point keeps its scratch (the per-row fp64 sums and 1/mean of
// tw_ternarize_pack) in a fixed array in device memory that is part of the
// loaded library: every GPU that loads the library holds those bytes until
// the process exits, and every call on that GPU shares them.
//
// The arithmetic is the same kernel sequence as tw_ternarize_pack.
#include <mutex>

#include "tw_device.cuh"
#include "tw_internal.h"

namespace {

// Scratch: 256 bytes for 1/mean, then one double per row.
constexpr int64_t kNoAllocMaxN = TW_NOALLOC_MAX_N;
constexpr size_t kNoAllocScratchBytes = 256 + 8 * (size_t)kNoAllocMaxN;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for the current device.  Host code
// must not pass the symbol itself to a kernel: on the host it names a
// stand-in object, not device memory.  Looked up once per device and
// context (again after a device reset, which creates a new context).
int scratch_address(void **out)
{
    static tw::SymbolCache cache;
    return tw::symbol_address(reinterpret_cast<const void *>(&g_noalloc_scratch), cache,
                              "no-alloc scratch", out);
}

}  // namespace

extern "C" TW_API int tw_ternarize_pack_noalloc(const float *W, int64_t N, int64_t K,
                                                void *packed, size_t packed_bytes,
                                                double *mean_abs, float *wscale,
                                                tw_stream_t stream)
{
    tw::clear_error();
    if (!W || !packed || !wscale)
        return tw::record_error(TW_ERR_NULL,
                                "tw_ternarize_pack_noalloc: W, packed and wscale are required");
    if (N < 1 || K < 1 || K % tw::kTileK)
        return tw::record_error(TW_ERR_SHAPE,
                                "tw_ternarize_pack_noalloc: need N >= 1 and K a positive "
                                "multiple of 128");
    if (N > kNoAllocMaxN)
        return tw::record_error(TW_ERR_SHAPE,
                                "tw_ternarize_pack_noalloc: N exceeds TW_NOALLOC_MAX_N (32768 "
                                "rows); use tw_ternarize_pack with a workspace");
    if (K > (1 << 24))
        return tw::record_error(TW_ERR_SHAPE, "tw_ternarize_pack_noalloc: K exceeds 2^24");
    const uintptr_t bad = reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(packed) |
                          reinterpret_cast<uintptr_t>(wscale) |
                          reinterpret_cast<uintptr_t>(mean_abs);
    if (bad & 15u)
        return tw::record_error(TW_ERR_ALIGN,
                                "tw_ternarize_pack_noalloc: pointers must be 16-byte aligned");
    if (packed_bytes < tw_packed_bytes(N, K))
        return tw::record_error(TW_ERR_BUFSIZE, "tw_ternarize_pack_noalloc: packed buffer too small");
    uint32_t *err = nullptr;
    if (int rc = tw::error_word(&err))
        return rc;
    void *scratch = nullptr;
    if (int rc = scratch_address(&scratch))
        return rc;
    // Every entry of the scratch that the kernels read is written first in
    // the same call (row sums, then 1/mean), so nothing needs clearing.
    cudaError_t e = tw::launch_ternarize(W, N, K, static_cast<uint8_t *>(packed), mean_abs,
                                         wscale, scratch, err, stream);
    if (e != cudaSuccess)
        return tw::record_error(TW_ERR_CUDA, cudaGetErrorString(e));
    return TW_OK;
}
