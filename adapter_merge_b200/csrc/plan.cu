// Plan construction and the host side of the C ABI: argument checks, the
// device table of linears, TMA descriptors (built once per plan), the work
// split of merge and apply, the device status word, and the entry points that
// launch the kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <new>

#include "internal.h"

namespace af {
namespace {

// The driver's tensor-map encoder, resolved once (thread-safe static
// initialisation); null if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// W-shaped map: 2-D [rows, cols] bf16 row-major, box 64 cols x box_rows rows,
// 128-byte swizzle.
bool encode_w(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows = 128)
{
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode_fn() && encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A stack: 3-D [E, r, d_in] bf16, box 64 (d_in) x rows x 1 (expert), 128-byte
// swizzle: a box is rows/8 whole 1 KB swizzle atoms of A rows.
bool encode_a(CUtensorMap* m, const void* ptr, int E, int r, int d_in, int64_t a_es, int rows, int experts = 1)
{
    cuuint64_t dims[3] = {(cuuint64_t)d_in, (cuuint64_t)r, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)d_in * 2, (cuuint64_t)a_es * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, (cuuint32_t)experts};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn() && encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B stack: 3-D [E, d_out, r] bf16, box 8 (r) x 128 (rows) x 1 (expert), no swizzle:
// one box is 16 stacked 8x8 core matrices (2 KB).
bool encode_b(CUtensorMap* m, const void* ptr, int E, int d_out, int r, int64_t b_es, int cols = 8)
{
    cuuint64_t dims[3] = {(cuuint64_t)r, (cuuint64_t)d_out, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)r * 2, (cuuint64_t)b_es * 2};
    cuuint32_t box[3] = {(cuuint32_t)cols, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : cols == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
    return encode_fn() && encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void free_plan(Plan* p)
{
    if (!p) return;
    if (p->d_desc) cudaFree(p->d_desc);
    if (p->d_maps) cudaFree(p->d_maps);
    if (p->d_status) cudaFree(p->d_status);
    for (int2* o : p->d_apply_order) if (o) cudaFree(o);
    if (p->d_sched) cudaFree(p->d_sched);
    if (p->d_call) cudaFree(p->d_call);
    delete static_cast<adafuse_plan*>(p);
}

}  // namespace
}  // namespace af

using namespace af;

extern "C" int adafuse_plan_create(adafuse_plan** out, const adafuse_linear* lins, int32_t n_lin, int32_t E,
                                   int32_t r, uint32_t flags)
{
    if (!out || !lins || n_lin < 1) return ADAFUSE_ERR_INVALID_ARG;
    *out = nullptr;
    if (E < 1 || E > kMaxE || r < 8 || r % 8 != 0 || r > kMaxKr) return ADAFUSE_ERR_UNSUPPORTED;
    if (flags & ~(ADAFUSE_PLAN_TEST_STALL | ADAFUSE_PLAN_Y_F32)) return ADAFUSE_ERR_INVALID_ARG;
    for (int l = 0; l < n_lin; ++l) {
        const adafuse_linear& L = lins[l];
        if (!L.W || !L.W_out || !L.A || !L.B) return ADAFUSE_ERR_INVALID_ARG;
        if (L.d_out < 8 || L.d_in < 8 || L.d_out % 8 || L.d_in % 8) return ADAFUSE_ERR_UNSUPPORTED;
        if (!aligned16(L.W) || !aligned16(L.W_out) || !aligned16(L.A) || !aligned16(L.B)) return ADAFUSE_ERR_UNSUPPORTED;
        if (L.a_expert_stride % 8 || L.b_expert_stride % 8) return ADAFUSE_ERR_UNSUPPORTED;
        if (L.a_expert_stride < (int64_t)r * L.d_in || L.b_expert_stride < (int64_t)L.d_out * r)
            return ADAFUSE_ERR_INVALID_ARG;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ADAFUSE_ERR_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ADAFUSE_ERR_DEVICE;
    if (prop.major != 10) return ADAFUSE_ERR_DEVICE;
    if (!encode_fn()) return ADAFUSE_ERR_CUDA;

    adafuse_plan* p = new (std::nothrow) adafuse_plan();
    if (!p) return ADAFUSE_ERR_CUDA;
    p->device = dev;
    p->num_sms = prop.multiProcessorCount;
    p->n_lin = n_lin;
    p->E = E;
    p->r = r;
    p->flags = flags;
    p->lins.assign(lins, lins + n_lin);
    p->h_desc.resize(n_lin);

    std::vector<CUtensorMap> maps((size_t)n_lin * kMapsPerLinear);
    p->a_box_rows = 8;
    while (p->a_box_rows < 128 && r % (2 * p->a_box_rows) == 0) p->a_box_rows *= 2;
    p->b_box_cols = r % 32 == 0 ? 32 : r % 16 == 0 ? 16 : 8;
    if (p->a_box_rows == r)
        while (2 * p->a_run_max <= E && 2 * p->a_run_max * r <= kTileM &&
               2 * p->a_run_max <= (2 << (kARunMaps - 1)))
            p->a_run_max *= 2;
    int64_t tiles = 0, units = 0;
    int32_t kslices[2] = {0, 0};
    for (int l = 0; l < n_lin; ++l) {
        const adafuse_linear& L = lins[l];
        LinDesc& d = p->h_desc[l];
        d.W = static_cast<const uint16_t*>(L.W);
        d.W_out = static_cast<uint16_t*>(L.W_out);
        d.A = static_cast<const uint16_t*>(L.A);
        d.B = static_cast<const uint16_t*>(L.B);
        d.a_es = L.a_expert_stride;
        d.b_es = L.b_expert_stride;
        d.d_out = L.d_out;
        d.d_in = L.d_in;
        d.n_rt = (L.d_out + kTileM - 1) / kTileM;
        d.n_strips = (L.d_in + kTileN - 1) / kTileN;
        d.tile_base = tiles;
        for (int g = 0; g < 2; ++g) {
            d.n_ks[g] = (L.d_in + shrink_ks(g) - 1) / shrink_ks(g);
            d.ks_base[g] = kslices[g];
            kslices[g] += d.n_ks[g];
        }
        tiles += (int64_t)d.n_rt * d.n_strips;
        units += d.n_rt;
        if (!encode_w(&maps[(size_t)l * kMapsPerLinear + kMapW], L.W, L.d_out, L.d_in) ||
            !encode_w(&maps[(size_t)l * kMapsPerLinear + kMapWout], L.W_out, L.d_out, L.d_in) ||
            !encode_w(&maps[(size_t)l * kMapsPerLinear + kMapWoutStore], L.W_out, L.d_out, L.d_in, 32) ||
            !encode_b(&maps[(size_t)l * kMapsPerLinear + kMapB], L.B, E, L.d_out, r, L.b_expert_stride) ||
            !encode_a(&maps[(size_t)l * kMapsPerLinear + kMapA], L.A, E, r, L.d_in, L.a_expert_stride, p->a_box_rows)) {
            free_plan(p);
            return ADAFUSE_ERR_UNSUPPORTED;
        }
        if ((r % 16 == 0 && !encode_b(&maps[(size_t)l * kMapsPerLinear + kMapB16], L.B, E, L.d_out, r,
                                      L.b_expert_stride, 16)) ||
            (r % 32 == 0 && !encode_b(&maps[(size_t)l * kMapsPerLinear + kMapB32], L.B, E, L.d_out, r,
                                      L.b_expert_stride, 32))) {
            free_plan(p);
            return ADAFUSE_ERR_UNSUPPORTED;
        }
        for (int i = 0; i < kARunMaps && (2 << i) <= p->a_run_max; ++i)
            if (!encode_a(&maps[(size_t)l * kMapsPerLinear + kMapARun + i], L.A, E, r, L.d_in, L.a_expert_stride,
                          p->a_box_rows, 2 << i)) {
                free_plan(p);
                return ADAFUSE_ERR_UNSUPPORTED;
            }
    }
    if (units > 0x7fffffff) { free_plan(p); return ADAFUSE_ERR_UNSUPPORTED; }
    p->merge_tiles = tiles;
    p->total_ks[0] = kslices[0];
    p->total_ks[1] = kslices[1];

    // Apply units, one list per unit height (H row blocks of 128), in
    // decreasing order of the W bytes they stream (stable), so that dynamic
    // scheduling ends with short units.
    std::vector<int2> order[kApplyShapes];
    for (int h = 0; h < kApplyShapes; ++h) {
        const int rows = kTileM << h;
        for (int l = 0; l < n_lin; ++l)
            for (int m = 0; m < (p->h_desc[l].d_out + rows - 1) / rows; ++m) order[h].push_back(make_int2(l, m));
        std::stable_sort(order[h].begin(), order[h].end(), [&](const int2& x, const int2& y) {
            return p->h_desc[x.x].d_in > p->h_desc[y.x].d_in;
        });
        p->apply_units[h] = (int64_t)order[h].size();
    }

    bool ok = cudaMalloc(&p->d_desc, sizeof(LinDesc) * n_lin) == cudaSuccess &&
              cudaMalloc(&p->d_maps, sizeof(CUtensorMap) * maps.size()) == cudaSuccess &&
              cudaMalloc(&p->d_status, sizeof(int32_t)) == cudaSuccess &&
              cudaMalloc(&p->d_sched, sizeof(int32_t) * 8) == cudaSuccess &&
              cudaMalloc(&p->d_call, apply_call_bytes(n_lin)) == cudaSuccess;
    for (int h = 0; h < kApplyShapes; ++h)
        ok = ok && cudaMalloc(&p->d_apply_order[h], sizeof(int2) * order[h].size()) == cudaSuccess &&
             cudaMemcpy(p->d_apply_order[h], order[h].data(), sizeof(int2) * order[h].size(),
                        cudaMemcpyHostToDevice) == cudaSuccess;
    ok = ok && cudaMemcpy(p->d_desc, p->h_desc.data(), sizeof(LinDesc) * n_lin, cudaMemcpyHostToDevice) == cudaSuccess;
    ok = ok && cudaMemcpy(p->d_maps, maps.data(), sizeof(CUtensorMap) * maps.size(), cudaMemcpyHostToDevice) == cudaSuccess;
    ok = ok && cudaMemset(p->d_sched, 0, sizeof(int32_t) * 8) == cudaSuccess;
    ok = ok && cudaMemset(p->d_status, 0, sizeof(int32_t)) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) { free_plan(p); return ADAFUSE_ERR_CUDA; }
    *out = p;
    return ADAFUSE_OK;
}

extern "C" void adafuse_plan_destroy(adafuse_plan* plan)
{
    if (!plan) return;
    cudaDeviceSynchronize();
    free_plan(plan);
}

static int check_sel(const adafuse_plan* p, const int32_t* idx, const float* gate, int32_t k, int ns)
{
    if (!p || !idx || !gate) return ADAFUSE_ERR_INVALID_ARG;
    if (k < 1 || k > p->E || ns > kMaxSlots || (int64_t)ns * p->r > kMaxKr) return ADAFUSE_ERR_UNSUPPORTED;
    return ADAFUSE_OK;
}

extern "C" int adafuse_merge(adafuse_plan* plan, const int32_t* idx, const float* gate, int32_t k,
                             adafuse_stream_t stream)
{
    int rc = check_sel(plan, idx, gate, k, k);
    if (rc) return rc;
    return launch_merge_fused(plan, idx, gate, nullptr, nullptr, k, 0, (cudaStream_t)stream);
}

extern "C" int adafuse_switch(adafuse_plan* plan, const int32_t* idx_new, const float* gate_new,
                              const int32_t* idx_old, const float* gate_old, int32_t k, adafuse_stream_t stream)
{
    int rc = check_sel(plan, idx_new, gate_new, k, 2 * k);
    if (rc) return rc;
    if (!idx_old || !gate_old) return ADAFUSE_ERR_INVALID_ARG;
    return launch_merge_fused(plan, idx_new, gate_new, idx_old, gate_old, k, 1, (cudaStream_t)stream);
}

extern "C" int adafuse_merge_per_linear(adafuse_plan* plan, const int32_t* idx, const float* gate, int32_t k,
                                        adafuse_stream_t stream)
{
    int rc = check_sel(plan, idx, gate, k, k);
    if (rc) return rc;
    return launch_merge_per_linear(plan, idx, gate, k, (cudaStream_t)stream);
}

extern "C" size_t adafuse_apply_workspace_bytes(const adafuse_plan* plan, int64_t T, int32_t k)
{
    if (!plan || T < 1 || k < 1) return 0;
    return apply_workspace_bytes(plan, T, k);
}

extern "C" int adafuse_apply(adafuse_plan* plan, const void* const* x_ptrs, void* const* y_ptrs, int64_t T,
                             const int32_t* idx, const float* gate, int32_t k, void* workspace, size_t ws_bytes,
                             adafuse_stream_t stream)
{
    if (!plan || !x_ptrs || !y_ptrs || !idx || !gate || !workspace || T < 1) return ADAFUSE_ERR_INVALID_ARG;
    if (k < 1 || k > plan->E) return ADAFUSE_ERR_UNSUPPORTED;
    if (T * (int64_t)k > 0x7fffffff) return ADAFUSE_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ADAFUSE_ERR_INVALID_ARG;
    return launch_apply(plan, x_ptrs, y_ptrs, T, idx, gate, k, workspace, ws_bytes, (cudaStream_t)stream);
}

extern "C" int adafuse_plan_status(adafuse_plan* plan, adafuse_stream_t stream, int32_t* device_status)
{
    if (!plan || !device_status) return ADAFUSE_ERR_INVALID_ARG;
    int32_t v = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ADAFUSE_ERR_CUDA;
    if (cudaMemcpy(&v, plan->d_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return ADAFUSE_ERR_CUDA;
    if (cudaMemset(plan->d_status, 0, sizeof(v)) != cudaSuccess) return ADAFUSE_ERR_CUDA;
    *device_status = v;
    return (v & ADAFUSE_STATUS_TIMEOUT) ? ADAFUSE_ERR_TIMEOUT : ADAFUSE_OK;
}

extern "C" int32_t adafuse_plan_last_launches(const adafuse_plan* plan)
{
    return plan ? plan->last_launches : 0;
}

extern "C" const char* adafuse_strerror(int code)
{
    switch (code) {
        case ADAFUSE_OK: return "ok";
        case ADAFUSE_ERR_INVALID_ARG: return "invalid argument";
        case ADAFUSE_ERR_UNSUPPORTED: return "unsupported shape, alignment or parameter";
        case ADAFUSE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case ADAFUSE_ERR_CUDA: return "CUDA runtime or driver error";
        case ADAFUSE_ERR_TIMEOUT: return "device-side wait timed out";
        case ADAFUSE_ERR_DEVICE: return "no usable sm_100 device";
        default: return "unknown error";
    }
}

extern "C" int32_t adafuse_version(void) { return 100; }
