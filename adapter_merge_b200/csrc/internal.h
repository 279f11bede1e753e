// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>
#include <vector>

#include "adafuse.h"

namespace af {

// One targeted linear as the kernels see it (device table, built once).
struct LinDesc {
    const uint16_t* W;
    uint16_t* W_out;
    const uint16_t* A;
    const uint16_t* B;
    int64_t a_es;          // expert stride of A, elements
    int64_t b_es;          // expert stride of B, elements
    int64_t tile_base;     // first merge tile (128 x 128) of this linear
    int32_t d_out, d_in;
    int32_t n_rt;          // ceil(d_out / 128)
    int32_t n_strips;      // ceil(d_in / 128)
    int32_t ks_base[2];    // first shrink K-slice of this linear, slices of shrink_ks(g) columns
    int32_t n_ks[2];       // ceil(d_in / shrink_ks(g))
};

// Tensor maps kept per linear: W (load, 64x128 boxes), W_out (load, 64x128
// boxes), B (3-D stack, 8x128x1 boxes), W_out store (64x32 boxes: one per
// merge epilogue warp), A (3-D stack, 64 x a_box_rows x 1 boxes, 128-byte
// swizzle) and, where a_box_rows == r, the A stack again in boxes of 2, 4, 8
// and 16 whole experts (kMapARun + i holds 2 << i experts), so that a run of
// consecutive experts moves in one load; where 16 (32) divides r, the B
// stack again in 16 x 128 boxes with 32-byte swizzle (32 x 128, 64-byte
// swizzle) for the apply's expand.
constexpr int kMapsPerLinear = 11;
constexpr int kMapW = 0, kMapWout = 1, kMapB = 2, kMapWoutStore = 3, kMapA = 4, kMapARun = 5;
constexpr int kMapB16 = 9, kMapB32 = 10;
constexpr int kARunMaps = 4;
// d_in columns per shrink work unit: g = 0 normally, g = 1 when the wide
// slices leave SMs idle
__host__ __device__ constexpr int shrink_ks(int g) { return g ? 256 : 1024; }

constexpr int kTileM = 128;      // output rows per tile (MMA M, TMEM lanes)
constexpr int kTileN = 128;      // merge: d_in columns per tile (MMA N)
constexpr int kChunkK = 64;      // apply: d_in per pipeline stage (one 128-byte swizzle row)
constexpr int kMaxSlots = ADAFUSE_MAX_SLOTS;
constexpr int kMaxKr = ADAFUSE_MAX_KR;
constexpr int kMaxE = ADAFUSE_MAX_E;
// Apply units cover H = 1, 2 or 4 row blocks of 128 (the MMAs of a unit share
// each x chunk); a unit of H blocks takes at most 256 / H tokens per tile, so
// that its two accumulators fit the 512 TMEM columns.
constexpr int kApplyShapes = 3;                   // H = 1 << shape

struct Plan {
    int device = 0;
    int num_sms = 0;
    int n_lin = 0, E = 0, r = 0;
    uint32_t flags = 0;
    std::vector<adafuse_linear> lins;
    std::vector<LinDesc> h_desc;
    LinDesc* d_desc = nullptr;
    CUtensorMap* d_maps = nullptr;
    int32_t* d_status = nullptr;
    int64_t merge_tiles = 0;
    int64_t apply_units[kApplyShapes] = {};       // apply units for H = 1, 2, 4
    int32_t total_ks[2] = {};         // shrink K-slices over all linears, per slice width
    int32_t a_box_rows = 8;           // rows per A-stack TMA box: largest power of two <= 128 dividing r
    int32_t a_run_max = 1;            // most experts one A-stack load may carry (1: no run maps)
    int32_t b_box_cols = 8;           // columns per B-stack box of the apply's expand: 8, 16 or 32
    int2* d_apply_order[kApplyShapes] = {};      // apply units (linear, row block), longest first
    int32_t* d_sched = nullptr;         // work counters of the persistent kernels (zero between launches)
    int32_t last_launches = 0;
    // Per-call apply descriptors: TMA maps of every x_l and of the shrink
    // output, and the x / y pointer tables, rebuilt only when the caller's
    // pointers, T, k or workspace change (the shrink-output map's base and
    // extent follow T * k).
    uint8_t* d_call = nullptr;
    bool call_valid = false;
    int64_t call_T = 0;
    int32_t call_k = 0;
    const void* call_ws = nullptr;
    std::vector<const void*> call_x, call_y;
};

}  // namespace af

struct adafuse_plan : public af::Plan {};

namespace af {

// Launchers (defined in the .cu files).  All return ADAFUSE_* codes.
int launch_merge_fused(Plan* p, const int32_t* idx0, const float* gate0, const int32_t* idx1,
                       const float* gate1, int32_t k, int mode, cudaStream_t s);
int launch_merge_per_linear(Plan* p, const int32_t* idx, const float* gate, int32_t k, cudaStream_t s);
int launch_segments(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offsets, int32_t* perm,
                    int32_t* used, int32_t* status, cudaStream_t s, int32_t* zero = nullptr, int64_t n_zero = 0);
size_t apply_workspace_bytes(const Plan* p, int64_t T, int32_t k);
size_t apply_call_bytes(int n_lin);
int launch_apply(Plan* p, const void* const* x_ptrs, void* const* y_ptrs, int64_t T, const int32_t* idx,
                 const float* gate, int32_t k, void* ws, size_t ws_bytes, cudaStream_t s);

inline int cuda_err(cudaError_t e) { return e == cudaSuccess ? ADAFUSE_OK : ADAFUSE_ERR_CUDA; }

// Launches a kernel with programmatic stream serialization, so that its
// launch and shared-memory prologue overlap the tail of the previous kernel
// in the stream.  Only for kernels that call griddep_wait() before any
// access to global memory or TMEM.
template <typename... Params, typename... Args>
inline int launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      Args&&... args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_err(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}

}  // namespace af
