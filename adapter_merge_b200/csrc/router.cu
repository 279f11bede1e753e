// Token-level pre-gating router.
//
// AdaFuse, page pt section 2.A ("Arquitetura de Pre-Gating por Token") and
// page ja section 2.1: a single lightweight top-2 router at the first expanded
// layer decides, once per input token, which LoRA experts are active in every
// later layer ("decide once, apply everywhere").  With ADAFUSE_POOL_MEAN the
// decision is taken once for the mean of the rows (the "whole sentence" case of
// the lay summary, section "A Solucao", item 1).
//
// One CTA per decision.  Warp 0 lane e owns expert e: its logit is the fp32 sum
// of the products x_j * W_r[e, j] in ascending j (products rounded before the
// add), so the decision is a fixed function of the inputs.  Where the whole
// W_r (rows padded to H + 4 floats) and the x row fit in shared memory, both
// are staged with 16-byte cp.async copies before the chain starts, which then
// runs with no barrier.  Otherwise W_r streams through a 4-stage cp.async ring
// (three 256-column chunks ahead), with the whole x row staged first when it
// fits; for the pooled mean and larger rows, warps 1-3 stage the next chunk of
// x while warp 0 consumes the current one.  Softmax and top-k are warp shuffles over the lanes (ties to the lower
// index, NaN ranked last).
#include "internal.h"
#include "ptx.cuh"

namespace af {

namespace {

constexpr int kChunk = 256;          // columns of x and W_r per pipeline stage
constexpr int kStages = 4;           // W_r chunks in flight: kStages - 1 ahead
constexpr int kRouterThreads = 128;

__device__ __forceinline__ float bf16_at(const uint16_t* p) { return __uint_as_float((uint32_t)(*p) << 16); }

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Is (c1, z1, e1) ranked before (c0, z0, e0)?  Class 0 = finite or infinite
// logit, 1 = NaN, 2 = no expert / already taken.
__device__ __forceinline__ bool ranks_before(int c1, float z1, int e1, int c0, float z0, int e0)
{
    if (c1 != c0) return c1 < c0;
    if (c1 == 0 && z1 != z0) return z1 > z0;
    return e1 < e0;
}

// W_r rows in a stage are padded to kChunk + 4 floats: 16-byte aligned for
// vector reads, and lane e's reads start 4 banks after lane e-1's.
constexpr int kRowPad = kChunk + 4;
__host__ __device__ constexpr int stage_floats(int E) { return E * kRowPad + kChunk; }

__global__ void __launch_bounds__(kRouterThreads) pregate_kernel(const uint16_t* x, int64_t T, int32_t H,
                                                                  int64_t ldx, const float* Wr, const float* br,
                                                                  int32_t E, int32_t k, uint32_t flags,
                                                                  int32_t* idx, float* gate, int xfull, int w16)
{
    // xfull: 0 = x staged chunk by chunk, 1 = whole x row first, 2 = whole
    // W_r and whole x row first (no ring, no per-chunk barriers).
    extern __shared__ float rsm[];
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool pool = (flags & ADAFUSE_POOL_MEAN) != 0;
    const int64_t t = pool ? 0 : blockIdx.x;
    const int nchunks = (H + kChunk - 1) / kChunk;
    const int SF = stage_floats(E);

    // W_r columns of chunk c -> stage buffer (ws[e][jj], rows padded to kChunk+1).
    auto issue_w = [&](int c) {
        if (c < nchunks) {
            float* ws = rsm + (c % kStages) * SF;
            const int j0 = c * kChunk;
            const int n = min(kChunk, H - j0);
            if (w16) {
                // 16-byte copies: W_r rows start on 16-byte boundaries (H % 4 == 0)
                for (int id = tid; id < E * (kChunk / 4); id += kRouterThreads) {
                    const int e = id / (kChunk / 4), jj = (id - e * (kChunk / 4)) * 4;
                    if (jj < n) cp_async_16(smem_u32(ws + e * kRowPad + jj), Wr + (int64_t)e * H + j0 + jj);
                }
            } else {
                for (int id = tid; id < E * kChunk; id += kRouterThreads) {
                    const int e = id / kChunk, jj = id - e * kChunk;
                    if (jj < n) cp_async_4(smem_u32(ws + e * kRowPad + jj), Wr + (int64_t)e * H + j0 + jj);
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // x (or the column means of x) for chunk c -> stage buffer, threads t0.. step nt.
    auto load_x = [&](int c, int t0, int nt) {
        float* xs = rsm + (c % kStages) * SF + E * kRowPad;
        const int j0 = c * kChunk;
        for (int jj = t0; jj < kChunk; jj += nt) {
            const int j = j0 + jj;
            float v = 0.f;
            if (j < H) {
                if (pool) {
                    float acc = 0.f;
                    for (int64_t tt = 0; tt < T; ++tt) acc = __fadd_rn(acc, bf16_at(x + tt * ldx + j));
                    v = __fdiv_rn(acc, (float)T);
                } else {
                    v = bf16_at(x + t * ldx + j);
                }
            }
            xs[jj] = v;
        }
    };

    float z = 0.f;
    if (xfull == 2) {
        // W_r rows padded to H + 4 floats (16-byte aligned, lanes 4 banks apart)
        const int Hp = H + 4;
        float* wall = rsm;
        float* xall = rsm + (size_t)E * Hp;
        for (int id = tid; id < E * (H / 4); id += kRouterThreads) {
            const int e = id / (H / 4), jj = (id - e * (H / 4)) * 4;
            cp_async_16(smem_u32(wall + (size_t)e * Hp + jj), Wr + (int64_t)e * H + jj);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll 8
        for (int j = tid; j < H; j += kRouterThreads) xall[j] = bf16_at(x + t * ldx + j);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        if (warp != 0) return;
        if (lane < E) {
            const float* ws = wall + (size_t)lane * Hp;
            const int n4 = H & ~15;
            // Same order as the scalar loop: one product, one add, ascending j.
            for (int jj = 0; jj < n4; jj += 16) {
                float4 xv[4], wv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    xv[u] = *reinterpret_cast<const float4*>(xall + jj + 4 * u);
                    wv[u] = *reinterpret_cast<const float4*>(ws + jj + 4 * u);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    z = __fadd_rn(z, __fmul_rn(xv[u].x, wv[u].x));
                    z = __fadd_rn(z, __fmul_rn(xv[u].y, wv[u].y));
                    z = __fadd_rn(z, __fmul_rn(xv[u].z, wv[u].z));
                    z = __fadd_rn(z, __fmul_rn(xv[u].w, wv[u].w));
                }
            }
            for (int jj = n4; jj < H; ++jj) z = __fadd_rn(z, __fmul_rn(xall[jj], ws[jj]));
        }
    } else {
    float* xall = rsm + kStages * SF;          // [H] when xfull
    for (int c = 0; c < kStages - 1; ++c) issue_w(c);
    if (xfull) {
#pragma unroll 8
        for (int j = tid; j < H; j += kRouterThreads) xall[j] = bf16_at(x + t * ldx + j);
    } else {
        load_x(0, tid, kRouterThreads);
    }
    for (int c = 0; c < nchunks; ++c) {
        issue_w(c + kStages - 1);
        asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1) : "memory");
        __syncthreads();                       // chunk c is in shared memory
        if (warp == 0) {
            if (lane < E) {
                const float* ws = rsm + (c % kStages) * SF + lane * kRowPad;
                const float* xs = xfull ? xall + c * kChunk : rsm + (c % kStages) * SF + E * kRowPad;
                const int n = min(kChunk, H - c * kChunk);
                const int n4 = n & ~15;
                // Same order as the scalar loop: one product, one add, ascending j.
                for (int jj = 0; jj < n4; jj += 16) {
                    float4 xv[4], wv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        xv[u] = *reinterpret_cast<const float4*>(xs + jj + 4 * u);
                        wv[u] = *reinterpret_cast<const float4*>(ws + jj + 4 * u);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        z = __fadd_rn(z, __fmul_rn(xv[u].x, wv[u].x));
                        z = __fadd_rn(z, __fmul_rn(xv[u].y, wv[u].y));
                        z = __fadd_rn(z, __fmul_rn(xv[u].z, wv[u].z));
                        z = __fadd_rn(z, __fmul_rn(xv[u].w, wv[u].w));
                    }
                }
                for (int jj = n4; jj < n; ++jj) z = __fadd_rn(z, __fmul_rn(xs[jj], ws[jj]));
            }
        } else if (!xfull && c + 1 < nchunks) {
            load_x(c + 1, tid - 32, kRouterThreads - 32);
        }
        __syncthreads();                       // stage c % kStages may be refilled
    }
    }
    if (warp != 0) return;

    if (lane < E && br != nullptr) z = __fadd_rn(z, br[lane]);
    const int cls = (lane >= E) ? 2 : (isnan(z) ? 1 : 0);

    // softmax over the experts with a non-NaN logit
    float m = (cls == 0) ? z : -INFINITY;
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float ex = (cls == 0) ? expf(z - m) : 0.f;
    float sum = ex;
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float p = ex / sum;

    // top-k by repeated warp argmax
    bool taken = false;
    int sel = 0;
    float gsel = 0.f, gsum = 0.f;
    for (int s = 0; s < k; ++s) {
        int bc = taken ? 2 : cls, be = lane;
        float bz = z;
        for (int off = 16; off > 0; off >>= 1) {
            const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
            const float oz = __shfl_xor_sync(0xffffffffu, bz, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ranks_before(oc, oz, oe, bc, bz, be)) { bc = oc; bz = oz; be = oe; }
        }
        if (lane == be) taken = true;
        const float pb = __shfl_sync(0xffffffffu, p, be);
        if (lane == s) { sel = be; gsel = pb; }
        gsum = __fadd_rn(gsum, pb);
    }
    if (lane < k) {
        float g = gsel;
        if (flags & ADAFUSE_RENORM) g = g / gsum;
        idx[t * k + lane] = sel;
        gate[t * k + lane] = g;
    }
}

}  // namespace
}  // namespace af

extern "C" int adafuse_pregate(const void* x, int64_t T, int32_t H, int64_t x_row_stride, const float* W_r,
                               const float* b_r, int32_t E, int32_t k, uint32_t flags, int32_t* idx, float* gate,
                               adafuse_stream_t stream)
{
    if (!x || !W_r || !idx || !gate || T < 1 || H < 1 || x_row_stride < H) return ADAFUSE_ERR_INVALID_ARG;
    if (E < 1 || E > af::kMaxE || k < 1 || k > E) return ADAFUSE_ERR_UNSUPPORTED;
    if (flags & ~(ADAFUSE_RENORM | ADAFUSE_POOL_MEAN)) return ADAFUSE_ERR_INVALID_ARG;
    const bool pool = (flags & ADAFUSE_POOL_MEAN) != 0;
    if (!pool && T > 0x7fffffff) return ADAFUSE_ERR_UNSUPPORTED;
    const unsigned grid = pool ? 1u : (unsigned)T;
    const int w16 = (H % 4 == 0 && (reinterpret_cast<uintptr_t>(W_r) & 15u) == 0) ? 1 : 0;
    size_t smem = sizeof(float) * af::kStages * af::stage_floats(E);
    const size_t smem_x = smem + sizeof(float) * (size_t)H;
    const size_t smem_all = sizeof(float) * ((size_t)E * (H + 4) + (size_t)H);
    int xfull = 0;
    if (!pool && w16 && smem_all <= 200 * 1024) { xfull = 2; smem = smem_all; }      // whole W_r and x
    else if (!pool && smem_x <= 200 * 1024) { xfull = 1; smem = smem_x; }            // whole x row
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(af::pregate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return ADAFUSE_ERR_CUDA;
    return af::launch_pdl(af::pregate_kernel, dim3(grid), dim3(af::kRouterThreads), smem, (cudaStream_t)stream,
                          static_cast<const uint16_t*>(x), T, H, x_row_stride, W_r, b_r, E, k, flags, idx, gate,
                          xfull, w16);
}
