// Fused all-layer LoRA merge (SGMM), its in-place switch variant, and the
// per-linear baseline.
//
// AdaFuse, page pt section 2.B ("Fusao de Adaptadores e Kernel SGMM") and page
// ja section 2.2: the activated adapters' down (A) and up (B) projections are
// concatenated and fused into the backbone weight of every targeted linear,
// W' = W + sum_s g_s B_{e_s} A_{e_s}, in a single kernel launch across layers,
// with the large product split into GEMM tiles assigned to thread blocks and a
// prefetch buffer hiding global->shared latency.
//
// B200 design: one persistent CTA per SM, warp-specialised, two variants.
//   merge_rows_kernel (k*r <= 128, every model configuration): 128 x 128
//     tiles walked along the rows of W in groups of 1, 2, 4 or 8 row blocks
//     interleaved column by column.  Warp 0 loads W tiles by TMA (two
//     64-column boxes, 128-byte swizzle) and, once per column block of a
//     group, the raw A rows of the selected experts (MN-major, 128-byte
//     swizzle) that all the group's tiles share; warps 2-3 load the selected
//     experts' B rows of the group's blocks by TMA and scale them by the
//     gates in place (Bcat, K-major core matrices); warp 1 issues tcgen05.mma
//     (dW = Bcat[128 x Kp] * Acat[Kp x 128], K = k*r) into one of two TMEM
//     accumulators of 128 columns.
//   merge_fused_kernel (k*r up to 256): tiles walked down 128-column strips;
//     the raw A rows of each strip come by TMA and warps 2-3 scale them by
//     the gates in place (Acat, MN-major, 128-byte swizzle), the B rows of
//     each tile come by TMA.
//   In both, warps 4-11 are the epilogue: each warp takes a 32-row x 64-column
//   slice: dW from TMEM (tcgen05.ld), W from the swizzled smem tile, W + dW
//   rounded to bf16 in place, and a TMA store of the slice.  A W stage is
//   released once the MMA and all eight stores have read it.
// HBM traffic is W read + W' write (4 bytes per element) plus the selected
// adapters; the tensor cores carry the rank-(k*r) contraction (16*k*r/4 FLOP/B).
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace af {

namespace {

struct MergeArgs {
    const LinDesc* lins;
    const CUtensorMap* maps;
    const int32_t* idx0;
    const float* gate0;
    const int32_t* idx1;
    const float* gate1;
    int32_t* status;
    int64_t total_tiles;
    int32_t n_lin;
    int32_t E, r;
    int32_t k;          // slots per selection
    int32_t ns;         // slots in this pass: k (merge) or 2k (switch)
    int32_t Kp;         // ns*r rounded up to 16
    int32_t mode;       // 0: merge W -> W_out; 1: switch, W_out in place
    int32_t stall;      // test hook: CTA 0 withholds its first W stage
    int32_t SW, SB, NA; // W stages, B stages, A buffers (row-order kernel: SB unused, NA = Bcat row blocks)
    int32_t NAR;        // row-order kernel: A tile slots
    int32_t G;          // row-order kernel: 128-row blocks per group
    int32_t box_rows;   // rows per A-stack TMA box (row-order kernel)
    uint32_t off_B, off_A, off_bar, stage_bytes;
};

constexpr int kMergeThreads = 384;
constexpr int kMergeThreadsTB = 448;     // row kernel with Bcat in TMEM: two more builder warps
constexpr uint32_t kWTileBytes = kTileM * kTileN * 2;       // 32 KB
constexpr uint32_t kWBoxBytes = kWTileBytes / 2;            // 16 KB: 64 cols x 128 rows
constexpr int kEpiWarps = 8;

struct TileIt {
    int l, strip, rt, n_rt, n_strips;
    __device__ void init(const LinDesc* lins, int n_lin, int64_t g)
    {
        int lo = 0, hi = n_lin - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (lins[mid].tile_base <= g) lo = mid; else hi = mid - 1;
        }
        l = lo;
        n_rt = lins[l].n_rt;
        n_strips = lins[l].n_strips;
        int64_t local = g - lins[l].tile_base;
        strip = (int)(local / n_rt);
        rt = (int)(local - (int64_t)strip * n_rt);
    }
    __device__ void next(const LinDesc* lins, int n_lin)
    {
        if (++rt == n_rt) {
            rt = 0;
            if (++strip == n_strips) {
                strip = 0;
                if (++l < n_lin) {
                    n_rt = lins[l].n_rt;
                    n_strips = lins[l].n_strips;
                }
            }
        }
    }
};

// Wait that ignores the abort flag (used to drain in-flight async work).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

__device__ __forceinline__ uint4 scale_bf16x8(uint4 raw, float g)
{
    uint4 o;
    o.x = pack_bf16x2(bf16lo(raw.x) * g, bf16hi(raw.x) * g);
    o.y = pack_bf16x2(bf16lo(raw.y) * g, bf16hi(raw.y) * g);
    o.z = pack_bf16x2(bf16lo(raw.z) * g, bf16hi(raw.z) * g);
    o.w = pack_bf16x2(bf16lo(raw.w) * g, bf16hi(raw.w) * g);
    return o;
}

__device__ __forceinline__ uint32_t add_bf16x2(uint32_t w, uint32_t d0, uint32_t d1)
{
    return pack_bf16x2(bf16lo(w) + __uint_as_float(d0), bf16hi(w) + __uint_as_float(d1));
}

// The selection into shared memory (one thread): s_e / s_g per slot, the old
// selection negated in switch mode; out-of-range expert ids become zero-gate
// empty slots and are flagged.  *s_skip = 1 for a switch between identical
// selections.
__device__ void read_selection(const MergeArgs& a, int* s_e, float* s_g, int* s_skip)
{
    int bad = 0;
    int same = 1;
    for (int s = 0; s < a.ns; ++s) {
        int e;
        float g;
        if (s < a.k) { e = a.idx0[s]; g = a.gate0[s]; }
        else { e = a.idx1[s - a.k]; g = -a.gate1[s - a.k]; }
        if (e < 0 || e >= a.E) { bad = 1; e = -1; g = 0.f; }
        s_e[s] = e;
        s_g[s] = g;
    }
    if (a.mode == 1) {
        for (int s = 0; s < a.k; ++s)
            if (a.idx0[s] != a.idx1[s] || __float_as_uint(a.gate0[s]) != __float_as_uint(a.gate1[s])) same = 0;
    } else {
        same = 0;
    }
    *s_skip = same;
    if (bad && blockIdx.x == 0) atomicOr(a.status, ADAFUSE_STATUS_BAD_INDEX);
}

__global__ void __launch_bounds__(kMergeThreads, 1) merge_fused_kernel(const __grid_constant__ MergeArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sW = base;
    uint8_t* sB = base + a.off_B;
    uint8_t* sA = base + a.off_A;
    uint64_t* wfull = reinterpret_cast<uint64_t*>(base + a.off_bar);
    uint64_t* wempty = wfull + a.SW;
    uint64_t* bfull = wempty + a.SW;
    uint64_t* bempty = bfull + a.SB;
    uint64_t* afull = bempty + a.SB;
    uint64_t* aempty = afull + a.NA;
    uint64_t* accfull = aempty + a.NA;
    uint64_t* accempty = accfull + 2;
    uint64_t* donebar = accempty + 2;
    uint64_t* aload = donebar + 1;                // raw A rows of a strip slot landed (TMA)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aload + a.NA);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_skip = reinterpret_cast<int*>(tmem_slot + 2);
    int* s_e = reinterpret_cast<int*>(tmem_slot + 4);
    float* s_g = reinterpret_cast<float*>(s_e + kMaxSlots);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t BBytes = (uint32_t)a.Kp * 256u;     // 128 rows x Kp bf16
    const uint32_t ABytes = (uint32_t)a.Kp * 256u;     // Kp rows x 128 cols bf16

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.SW; ++i) { mbar_init(&wfull[i], 1); mbar_init(&wempty[i], kEpiWarps); }
        for (int i = 0; i < a.SB; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
        for (int i = 0; i < a.NA; ++i) { mbar_init(&afull[i], 2); mbar_init(&aempty[i], 1); mbar_init(&aload[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], kEpiWarps); }
        mbar_init(donebar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Zero the B ring and the A strip slots: stages of skipped slots and the
    // K padding are never loaded and stay zero.
    for (uint32_t o = threadIdx.x * 16; o < (uint32_t)a.SB * BBytes; o += kMergeThreads * 16)
        st_shared_v4(smem_u32(sB + o), make_uint4(0, 0, 0, 0));
    for (uint32_t o = threadIdx.x * 16; o < (uint32_t)a.NA * ABytes; o += kMergeThreads * 16)
        st_shared_v4(smem_u32(sA + o), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x == 0) read_selection(a, s_e, s_g, s_skip);
    __syncthreads();
    if (*s_skip) return;       // switch between identical selections: nothing to do

    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t t_begin = (int64_t)blockIdx.x * a.total_tiles / G;
    const int64_t t_end = ((int64_t)blockIdx.x + 1) * a.total_tiles / G;
    const int64_t count = t_end - t_begin;
    const int kmap_in = a.mode == 1 ? kMapWout : kMapW;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && count > 0) {
            TileIt it;
            it.init(a.lins, a.n_lin, t_begin);
            int nbox = 0;
            for (int s = 0; s < a.ns; ++s) if (s_e[s] >= 0) nbox += a.r / 8;
            const uint32_t bbytes = (uint32_t)nbox * 2048u;
            int64_t issued_w = 0, issued_b = 0;
            for (int64_t i = 0; i < count; ++i) {
                const int sw = (int)(i % a.SW);
                if (!mbar_wait(&wempty[sw], (uint32_t)((i / a.SW) & 1) ^ 1u, abort_flag)) break;
                const CUtensorMap* mW = a.maps + (size_t)it.l * kMapsPerLinear + kmap_in;
                const int n0 = it.strip * kTileN, m0 = it.rt * kTileM;
                uint8_t* dstW = sW + (size_t)sw * kWTileBytes;
                if (!(a.stall && blockIdx.x == 0 && i == 0)) {
                    mbar_arrive_expect_tx(&wfull[sw], kWTileBytes);
                    tma_load_2d(dstW, mW, &wfull[sw], n0, m0);
                    tma_load_2d(dstW + kWBoxBytes, mW, &wfull[sw], n0 + 64, m0);
                    issued_w = i + 1;
                }

                const int sb = (int)(i % a.SB);
                if (!mbar_wait(&bempty[sb], (uint32_t)((i / a.SB) & 1) ^ 1u, abort_flag)) break;
                const CUtensorMap* mB = a.maps + (size_t)it.l * kMapsPerLinear + kMapB;
                uint8_t* dstB = sB + (size_t)sb * BBytes;
                mbar_arrive_expect_tx(&bfull[sb], bbytes);
                for (int s = 0; s < a.ns; ++s) {
                    const int e = s_e[s];
                    if (e < 0) continue;
                    for (int jg = 0; jg < a.r / 8; ++jg)
                        tma_load_3d(dstB + (size_t)((s * a.r) / 8 + jg) * 2048u, mB, &bfull[sb], jg * 8, m0, e);
                }
                issued_b = i + 1;
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            // Drain: the loads this thread issued must land before the CTA exits.
            for (int64_t j = std::max<int64_t>(0, issued_w - a.SW); j < issued_w; ++j)
                mbar_wait_drain(&wfull[j % a.SW], (uint32_t)((j / a.SW) & 1));
            for (int64_t j = std::max<int64_t>(0, issued_b - a.SB); j < issued_b; ++j)
                mbar_wait_drain(&bfull[j % a.SB], (uint32_t)((j / a.SB) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && count > 0) {
            TileIt it;
            it.init(a.lins, a.n_lin, t_begin);
            const uint32_t idesc = make_idesc_bf16(kTileM, kTileN, 0u, 1u);
            const uint32_t lbo_a = (uint32_t)a.Kp * 128u;    // 64-column halves of the A strip
            int64_t strip_seq = -1;
            for (int64_t i = 0; i < count; ++i) {
                const bool first = (i == 0) || (it.rt == 0);
                const bool last = (i + 1 == count) || (it.rt == it.n_rt - 1);
                if (first) ++strip_seq;
                const int ab = (int)(strip_seq % a.NA);
                const int sb = (int)(i % a.SB);
                const int acc = (int)(i & 1);
                if (!mbar_wait(&bfull[sb], (uint32_t)((i / a.SB) & 1), abort_flag)) break;
                if (first && !mbar_wait(&afull[ab], (uint32_t)((strip_seq / a.NA) & 1), abort_flag)) break;
                if (!mbar_wait(&accempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)acc * kTileN;
                const uint32_t baddr = smem_u32(sB + (size_t)sb * BBytes);
                const uint32_t aaddr = smem_u32(sA + (size_t)ab * ABytes);
                for (int kk = 0; kk < a.Kp / 16; ++kk) {
                    const uint64_t adesc = make_sdesc(baddr + (uint32_t)kk * 4096u, 2048u, 128u, kLayoutNone);
                    const uint64_t bdesc = make_sdesc(aaddr + (uint32_t)kk * 2048u, lbo_a, 1024u, kLayoutSw128);
                    tc_mma_bf16(d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                }
                tc_commit(&accfull[acc]);
                tc_commit(&bempty[sb]);
                if (last) tc_commit(&aempty[ab]);
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            tc_commit(donebar);
            mbar_wait_drain(donebar, 0);
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------ Acat builder
        // The raw A rows of the selected experts for the strip's 128 columns
        // come by TMA (3-D map over the expert stack, MN-major, 128-byte
        // swizzle: K row c of column half h at bytes h*Kp*128 + c*128), then
        // both warps scale each loaded row by its slot's gate in place.
        // Rows of skipped slots and the K padding are never loaded and stay
        // zero; columns past d_in arrive as zeros.
        if (count > 0) {
            const int tb = (warp - 2) * 32 + lane;
            TileIt it;
            it.init(a.lins, a.n_lin, t_begin);
            int nvalid = 0;
            for (int s2 = 0; s2 < a.ns; ++s2) if (s_e[s2] >= 0) ++nvalid;
            const uint32_t abytes = (uint32_t)nvalid * (uint32_t)a.r * 256u;     // 2 halves x r rows x 128 B
            const int R = a.box_rows;
            int64_t strip_seq = -1, loaded = -1;
            for (int64_t i = 0; i < count; ++i) {
                if (i == 0 || it.rt == 0) {
                    ++strip_seq;
                    const int ab = (int)(strip_seq % a.NA);
                    bool ok = mbar_wait(&aempty[ab], (uint32_t)((strip_seq / a.NA) & 1) ^ 1u, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const int n0 = it.strip * kTileN;
                    uint8_t* adst = sA + (size_t)ab * ABytes;
                    if (warp == 2 && lane == 0) {
                        const CUtensorMap* mA = a.maps + (size_t)it.l * kMapsPerLinear + kMapA;
                        mbar_arrive_expect_tx(&aload[ab], abytes);
                        for (int s2 = 0; s2 < a.ns; ++s2) {
                            const int e = s_e[s2];
                            if (e < 0) continue;
                            for (int h = 0; h < 2; ++h)
                                for (int j0 = 0; j0 < a.r; j0 += R)
                                    tma_load_3d(adst + (size_t)h * a.Kp * 128u + (size_t)((s2 * a.r + j0) / 8) * 1024u,
                                                mA, &aload[ab], n0 + 64 * h, j0, e);
                        }
                        loaded = strip_seq;
                    }
                    ok = mbar_wait(&aload[ab], (uint32_t)((strip_seq / a.NA) & 1), abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const int rowchunks = a.Kp * 8;               // 16-byte chunks per column half
                    const int chunks = 2 * rowchunks;
                    for (int id0 = tb; id0 < chunks; id0 += 4 * 64) {
                        uint4 v[4];
                        float gs[4];
                        bool slot[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int id = id0 + u * 64;
                            const int c = (id % rowchunks) >> 3;       // K row of the chunk
                            const int s2 = c / a.r;
                            slot[u] = id < chunks && s2 < a.ns && s_e[s2] >= 0;
                            gs[u] = slot[u] ? s_g[s2] : 0.f;
                            v[u] = slot[u] ? ld_shared_v4(smem_u32(adst) + (uint32_t)id * 16u) : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (slot[u]) st_shared_v4(smem_u32(adst) + (uint32_t)(id0 + u * 64) * 16u, scale_bf16x8(v[u], gs[u]));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&afull[ab]);
                }
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            // After an abort the last A loads may still be in flight.
            if (warp == 2 && lane == 0 && loaded >= 0)
                mbar_wait_drain(&aload[loaded % a.NA], (uint32_t)((loaded / a.NA) & 1));
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warp (q, h) owns rows 32q..32q+31 and columns 64h..64h+63 of the
        // tile: it reads that slice of dW from TMEM, adds it to the W slice in
        // shared memory, and stores the slice itself with one TMA store.  A W
        // stage is released (8 arrivals) once every warp's store has read it.
        const int ew = warp - 4;            // 0..7
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int h = ew >> 2;              // column half (64 columns)
        const int row = q * 32 + lane;
        TileIt it;
        if (count > 0) it.init(a.lins, a.n_lin, t_begin);
        int64_t stored = 0;
        for (int64_t i = 0; i < count; ++i) {
            const int acc = (int)(i & 1);
            const int sw = (int)(i % a.SW);
            bool ok = mbar_wait(&accfull[acc], (uint32_t)((i >> 1) & 1), abort_flag);
            ok = ok && mbar_wait(&wfull[sw], (uint32_t)((i / a.SW) & 1), abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t va[32], vb[32];
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * kTileN + (uint32_t)h * 64u;
            tc_ld_x32(taddr, va);
            tc_ld_x32(taddr + 32u, vb);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            uint8_t* slice = sW + (size_t)sw * kWTileBytes + (size_t)h * kWBoxBytes + (size_t)q * 32 * 128;
            const uint32_t wrow = smem_u32(slice) + (uint32_t)lane * 128u;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t addr = wrow + ((uint32_t)(c ^ (row & 7)) << 4);
                const uint4 w = ld_shared_v4(addr);
                const uint32_t* d = (c < 4) ? &va[c * 8] : &vb[(c - 4) * 8];
                uint4 o;
                o.x = add_bf16x2(w.x, d[0], d[1]);
                o.y = add_bf16x2(w.y, d[2], d[3]);
                o.z = add_bf16x2(w.z, d[4], d[5]);
                o.w = add_bf16x2(w.w, d[6], d[7]);
                st_shared_v4(addr, o);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const CUtensorMap* mO = a.maps + (size_t)it.l * kMapsPerLinear + kMapWoutStore;
                tma_store_2d(mO, slice, it.strip * kTileN + h * 64, it.rt * kTileM + q * 32);
                bulk_commit_group();
                bulk_wait_group_read<1>();
                if (i > 0) mbar_arrive(&wempty[(i - 1) % a.SW]);
            }
            stored = i + 1;
            if (i + 1 < count) it.next(a.lins, a.n_lin);
        }
        if (lane == 0) {
            bulk_wait_group<0>();
            if (stored > 0) mbar_arrive(&wempty[(stored - 1) % a.SW]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 256);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.status, ADAFUSE_STATUS_TIMEOUT);
}


// ------------------------------------------------------------------ row order

// Row-order variant (k*r <= 128).  Tiles are walked along the rows of W in
// groups of G (1, 2, 4 or 8) 128-row blocks, the blocks of a group interleaved
// column block by column block: (block 0, cols 0-127), (block 1, cols 0-127),
// ..., (block 0, cols 128-255), ...  Consecutive tiles of a CTA continue the
// same rows of W (long contiguous DRAM runs), and the raw A rows of a
// 128-column block (Kp x 128, MN-major, 128-byte swizzle, loaded by TMA into
// a ring of their own) serve all G blocks of the group: 1/G of the A traffic
// of walking one block at a time, where those loads cost 12 % of the launch.
// The gate sits on the B side: warps 2-3 build the gate-scaled Bcat of the
// group's blocks (128 rows x Kp each, K-major core matrices) once per group.
// A W stage is released by the MMA and the eight epilogue stores (W' read),
// an A slot by the MMA of its column block's last tile, a Bcat group slot by
// the MMA of the group's last tile.
struct GroupTileIt {
    int l, gi, strip, b, nb, n_rt, n_strips, G;
    __device__ int rt() const { return G * gi + b; }
    __device__ void set_nb() { nb = min(G, n_rt - G * gi); }
    __device__ void init(const LinDesc* lins, int n_lin, int64_t g, int group)
    {
        G = group;
        int lo = 0, hi = n_lin - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (lins[mid].tile_base <= g) lo = mid; else hi = mid - 1;
        }
        l = lo;
        n_rt = lins[l].n_rt;
        n_strips = lins[l].n_strips;
        const int64_t local = g - lins[l].tile_base;
        const int64_t group_tiles = (int64_t)G * n_strips;
        const int full_groups = n_rt / G;
        if (local < (int64_t)full_groups * group_tiles) {
            gi = (int)(local / group_tiles);
            const int rem = (int)(local - (int64_t)gi * group_tiles);
            strip = rem / G;
            b = rem - strip * G;
        } else {                                   // the blocks left when G does not divide n_rt
            gi = full_groups;
            const int left = n_rt - full_groups * G;
            const int rem = (int)(local - (int64_t)full_groups * group_tiles);
            strip = rem / left;
            b = rem - strip * left;
        }
        set_nb();
    }
    __device__ void next(const LinDesc* lins, int n_lin)
    {
        if (++b < nb) return;
        b = 0;
        if (++strip < n_strips) return;
        strip = 0;
        if (G * ++gi < n_rt) { set_nb(); return; }
        gi = 0;
        if (++l < n_lin) {
            n_rt = lins[l].n_rt;
            n_strips = lins[l].n_strips;
            set_nb();
        }
    }
    __device__ bool col_first() const { return b == 0; }
    __device__ bool col_last() const { return b == nb - 1; }
    __device__ bool group_first() const { return b == 0 && strip == 0; }
    __device__ bool group_last() const { return b == nb - 1 && strip == n_strips - 1; }
};

// Gate-scales the 16-byte chunks id = tid, tid + nthr, ... of a group's raw
// B rows in shared memory (chunk id: block, 8-column group, row; four chunks
// per step, their loads issued together); chunks of slots without an expert
// and of the K padding become zeros.
__device__ __forceinline__ void scale_bcat_chunks(uint8_t* gbase, int chunks, int groups, int r, int ns,
                                                  const int* s_e, const float* s_g, int tid, int nthr)
{
    for (int id0 = tid; id0 < chunks; id0 += 4 * nthr) {
        uint4 v[4];
        float gs[4];
        bool live[4], slot[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int id = id0 + u * nthr;
            const int cg = (id / kTileM) % groups;
            const int s2 = (cg * 8) / r;
            live[u] = id < chunks;
            slot[u] = live[u] && s2 < ns && s_e[s2] >= 0;
            gs[u] = slot[u] ? s_g[s2] : 0.f;
            v[u] = slot[u] ? ld_shared_v4(smem_u32(gbase) + (uint32_t)id * 16u) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (live[u])    // address = block*BcBytes + cg*2048 + row*16
                st_shared_v4(smem_u32(gbase) + (uint32_t)(id0 + u * nthr) * 16u,
                             slot[u] ? scale_bf16x8(v[u], gs[u]) : make_uint4(0, 0, 0, 0));
    }
}

template <bool kTB>
__global__ void __launch_bounds__(kTB ? kMergeThreadsTB : kMergeThreads, 1)
    merge_rows_kernel(const __grid_constant__ MergeArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sStage = base;                       // SW x W tile (32 KB)
    uint8_t* sA = base + a.off_A;                 // NAR x A tile [Kp x 128], MN-major, 128-byte swizzle
    uint8_t* sBcat = base + a.off_B;              // NA x [128 x Kp] gate-scaled B rows, G per group slot (smem Bcat)
    const int NP = a.NA / a.G;                    // Bcat group slots
    uint64_t* full = reinterpret_cast<uint64_t*>(base + a.off_bar);
    uint64_t* empty = full + a.SW;
    uint64_t* afull = empty + a.SW;
    uint64_t* aempty = afull + a.NAR;
    uint64_t* bcfull = aempty + a.NAR;
    uint64_t* bcempty = bcfull + NP;
    uint64_t* bcload = bcempty + NP;              // raw B rows of a group slot landed (TMA)
    uint64_t* accfull = bcload + NP;
    uint64_t* accempty = accfull + 2;
    uint64_t* donebar = accempty + 2;
    uint64_t* b0done = donebar + 1;               // (smem Bcat) the epilogue warps' share of the first group scaled
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b0done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_skip = reinterpret_cast<int*>(tmem_slot + 2);
    volatile int* s_bfirst = reinterpret_cast<volatile int*>(tmem_slot + 3);   // first B-row loads issued
    int* s_e = reinterpret_cast<int*>(tmem_slot + 4);
    float* s_g = reinterpret_cast<float*>(s_e + kMaxSlots);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t ATile = (uint32_t)a.Kp * 256u;      // Kp rows x 128 cols bf16
    const uint32_t BcBytes = (uint32_t)a.Kp * 256u;    // 128 rows x Kp bf16

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.SW; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], kEpiWarps + 1); }
        for (int i = 0; i < a.NAR; ++i) { mbar_init(&afull[i], 1); mbar_init(&aempty[i], 1); }
        for (int i = 0; i < NP; ++i) { mbar_init(&bcfull[i], kTB ? 4 : 2); mbar_init(&bcempty[i], 1); mbar_init(&bcload[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], kEpiWarps); }
        mbar_init(donebar, 1);
        mbar_init(b0done, kEpiWarps);
        *abort_flag = 0;
        *s_bfirst = 0;
        fence_mbar_init();
    }
    // Zero every A slot: the K padding rows and the rows of skipped slots are
    // never loaded and must read as finite zeros.
    for (int st = 0; st < a.NAR; ++st)
        for (uint32_t o = threadIdx.x * 16; o < ATile; o += blockDim.x * 16)
            st_shared_v4(smem_u32(sA + (size_t)st * ATile + o), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x == 0) read_selection(a, s_e, s_g, s_skip);
    __syncthreads();
    if (*s_skip) return;       // switch between identical selections: nothing to do

    // TMEM: two 128-column accumulators, then (kTB) the Bcat group slots,
    // Kp / 2 columns per row block.
    constexpr uint32_t kTmemCols = kTB ? 512u : 256u;
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t t_begin = (int64_t)blockIdx.x * a.total_tiles / G;
    const int64_t t_end = ((int64_t)blockIdx.x + 1) * a.total_tiles / G;
    const int64_t count = t_end - t_begin;
    const int kmap_in = a.mode == 1 ? kMapWout : kMapW;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && count > 0) {
            GroupTileIt it;
            it.init(a.lins, a.n_lin, t_begin, a.G);
            int nvalid = 0;
            for (int s = 0; s < a.ns; ++s) if (s_e[s] >= 0) ++nvalid;
            const uint32_t abytes = (uint32_t)nvalid * (uint32_t)a.r * 256u;    // 2 halves x r rows x 128 B
            const int R = a.box_rows;
            int64_t issued = 0, aseq = -1, a_issued = 0;
            // The SM's TMA engine serves requests in issue order: the first
            // group's B rows (issued by the Bcat builder) and the first A
            // tile go ahead of the W stream, so the first MMA does not wait
            // behind every W stage of the ring.
            if (!kTB) {                 // (B rows in TMEM come by plain loads)
                const uint64_t t0 = globaltimer_ns();
                while (!*s_bfirst && !*abort_flag) {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) { *abort_flag = 1; break; }
                }
            }
            for (int64_t i = 0; i < count; ++i) {
                const int sw = (int)(i % a.SW);
                if (!mbar_wait(&empty[sw], (uint32_t)((i / a.SW) & 1) ^ 1u, abort_flag)) break;
                const CUtensorMap* mW = a.maps + (size_t)it.l * kMapsPerLinear + kmap_in;
                const int n0 = it.strip * kTileN, m0 = it.rt() * kTileM;
                uint8_t* dst = sStage + (size_t)sw * a.stage_bytes;
                // The A rows of this column block, for every tile of the
                // group.  The first tile's go ahead of its W tile (the TMA
                // engine serves an SM's requests in issue order); later ones
                // follow their W tile, so a full A ring never holds up the W
                // stream.
                auto issue_a = [&]() -> bool {
                    const int as = (int)(++aseq % a.NAR);
                    if (!mbar_wait(&aempty[as], (uint32_t)((aseq / a.NAR) & 1) ^ 1u, abort_flag)) return false;
                    const CUtensorMap* mA = a.maps + (size_t)it.l * kMapsPerLinear + kMapA;
                    uint8_t* adst = sA + (size_t)as * ATile;
                    mbar_arrive_expect_tx(&afull[as], abytes);
                    for (int s = 0; s < a.ns; ++s) {
                        const int e = s_e[s];
                        if (e < 0) continue;
                        for (int h = 0; h < 2; ++h)
                            for (int j0 = 0; j0 < a.r; j0 += R)
                                tma_load_3d(adst + (size_t)h * a.Kp * 128u + (size_t)((s * a.r + j0) / 8) * 1024u,
                                            mA, &afull[as], n0 + 64 * h, j0, e);
                    }
                    a_issued = aseq + 1;
                    return true;
                };
                if (i == 0 && !issue_a()) break;
                if (!(a.stall && blockIdx.x == 0 && i == 0)) {
                    mbar_arrive_expect_tx(&full[sw], kWTileBytes);
                    tma_load_2d(dst, mW, &full[sw], n0, m0);
                    tma_load_2d(dst + kWBoxBytes, mW, &full[sw], n0 + 64, m0);
                    issued = i + 1;
                }
                if (i > 0 && it.col_first() && !issue_a()) break;
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            // Drain the TMA loads still in flight before the CTA may exit.
            for (int64_t j = std::max<int64_t>(0, issued - a.SW); j < issued; ++j)
                mbar_wait_drain(&full[j % a.SW], (uint32_t)((j / a.SW) & 1));
            for (int64_t j = std::max<int64_t>(0, a_issued - a.NAR); j < a_issued; ++j)
                mbar_wait_drain(&afull[j % a.NAR], (uint32_t)((j / a.NAR) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && count > 0) {
            GroupTileIt it;
            it.init(a.lins, a.n_lin, t_begin, a.G);
            const uint32_t idesc = make_idesc_bf16(kTileM, kTileN, 0u, 1u);
            const uint32_t lbo_a = (uint32_t)a.Kp * 128u;       // 64-column blocks of the A tile
            int64_t pseq = -1, aseq = -1;
            for (int64_t i = 0; i < count; ++i) {
                const bool pfirst = (i == 0) || it.group_first();
                const bool plast = (i + 1 == count) || it.group_last();
                const bool cfirst = (i == 0) || it.col_first();
                const bool clast = (i + 1 == count) || it.col_last();
                if (pfirst) ++pseq;
                if (cfirst) ++aseq;
                const int ps = (int)(pseq % NP), as = (int)(aseq % a.NAR);
                const int sw = (int)(i % a.SW);
                const int acc = (int)(i & 1);
                if (!mbar_wait(&full[sw], (uint32_t)((i / a.SW) & 1), abort_flag)) break;
                if (cfirst && !mbar_wait(&afull[as], (uint32_t)((aseq / a.NAR) & 1), abort_flag)) break;
                if (pfirst && !mbar_wait(&bcfull[ps], (uint32_t)((pseq / NP) & 1), abort_flag)) break;
                if (!mbar_wait(&accempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)acc * kTileN;
                const uint32_t bcaddr = smem_u32(sBcat + (size_t)(ps * a.G + it.b) * BcBytes);
                const uint32_t aaddr = smem_u32(sA + (size_t)as * ATile);
                const uint32_t bc_tmem = tmem_base + 256u + (uint32_t)((ps * a.G + it.b) * (a.Kp / 2));
                for (int kk = 0; kk < a.Kp / 16; ++kk) {
                    const uint64_t bdesc = make_sdesc(aaddr + (uint32_t)kk * 2048u, lbo_a, 1024u, kLayoutSw128);
                    if (kTB) {
                        tc_mma_bf16_ta(d, bc_tmem + (uint32_t)kk * 8u, bdesc, idesc, kk > 0 ? 1u : 0u);
                    } else {
                        const uint64_t adesc = make_sdesc(bcaddr + (uint32_t)kk * 4096u, 2048u, 128u, kLayoutNone);
                        tc_mma_bf16(d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                    }
                }
                tc_commit(&accfull[acc]);
                tc_commit(&empty[sw]);
                if (clast) tc_commit(&aempty[as]);
                if (plast) tc_commit(&bcempty[ps]);
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            tc_commit(donebar);
            mbar_wait_drain(donebar, 0);
        }
        __syncwarp();
    } else if (kTB && (warp == 2 || warp == 3 || warp >= 4 + kEpiWarps)) {
        // ------------------------------------------------------------ Bcat builder (TMEM)
        // Warps 2, 3, 12 and 13 cover TMEM lane quarters 2, 3, 0 and 1: each
        // lane loads its row's B values of every selected expert (16-byte
        // global loads), scales them by the slot's gate, packs them two bf16
        // per 32-bit column (lower K index in the low half) and stores them
        // into the group slot's TMEM columns; slots without an expert, the K
        // padding and rows past d_out are zeros.
        if (count > 0) {
            const int q = warp & 3;
            GroupTileIt it;
            it.init(a.lins, a.n_lin, t_begin, a.G);
            int64_t pseq = -1;
            for (int64_t i = 0; i < count; ++i) {
                if (i == 0 || it.group_first()) {
                    ++pseq;
                    const int ps = (int)(pseq % NP);
                    bool ok = mbar_wait(&bcempty[ps], (uint32_t)((pseq / NP) & 1) ^ 1u, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    const LinDesc& L = a.lins[it.l];
                    const uint16_t* Bp = L.B;
                    const int64_t b_es = L.b_es;
                    const int d_out = L.d_out;
                    for (int bq = 0; bq < it.nb; ++bq) {
                        const int row = (a.G * it.gi + bq) * kTileM + q * 32 + lane;
                        const uint32_t col0 = 256u + (uint32_t)((ps * a.G + bq) * (a.Kp / 2));
                        for (int k32 = 0; k32 < a.Kp / 32; ++k32) {
                            uint4 v[4];
#pragma unroll
                            for (int pc = 0; pc < 4; ++pc) {
                                const int c = k32 * 32 + pc * 8;          // 8 consecutive K of one slot
                                const int s2 = c / a.r, jj = c - s2 * a.r;
                                v[pc] = make_uint4(0, 0, 0, 0);
                                if (s2 < a.ns && s_e[s2] >= 0 && row < d_out)
                                    v[pc] = scale_bf16x8(ld_global_nc_v4(Bp + (int64_t)s_e[s2] * b_es + (int64_t)row * a.r + jj),
                                                         s_g[s2]);
                            }
                            const uint32_t w[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                                    v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
                            tc_st_x16(tmem_base + ((uint32_t)(q * 32) << 16) + col0 + (uint32_t)k32 * 16u, w);
                        }
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bcfull[ps]);
                }
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
        }
    } else if (!kTB && (warp == 2 || warp == 3)) {
        // ------------------------------------------------------------ Bcat builder
        if (count > 0) {
            const int tb = (warp - 2) * 32 + lane;
            GroupTileIt it;
            it.init(a.lins, a.n_lin, t_begin, a.G);
            int64_t pseq = -1, loaded = -1;
            for (int64_t i = 0; i < count; ++i) {
                if (i == 0 || it.group_first()) {
                    ++pseq;
                    const int ps = (int)(pseq % NP);
                    bool ok = mbar_wait(&bcempty[ps], (uint32_t)((pseq / NP) & 1) ^ 1u, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    // The raw B rows of every block of the group come by TMA
                    // (one 128-row x 8-column box per expert column group,
                    // already in the K-major core-matrix layout), then both
                    // warps scale them by their slot's gate in place; slots
                    // without an expert and the K padding become zeros.
                    uint8_t* gbase = sBcat + (size_t)ps * a.G * BcBytes;
                    if (warp == 2 && lane == 0) {
                        int nvalid = 0;
                        for (int s2 = 0; s2 < a.ns; ++s2) if (s_e[s2] >= 0) ++nvalid;
                        const CUtensorMap* mB = a.maps + (size_t)it.l * kMapsPerLinear + kMapB;
                        mbar_arrive_expect_tx(&bcload[ps], (uint32_t)(it.nb * nvalid * a.r) * 256u);
                        for (int bq = 0; bq < it.nb; ++bq)
                            for (int s2 = 0; s2 < a.ns; ++s2) {
                                const int e = s_e[s2];
                                if (e < 0) continue;
                                for (int j0 = 0; j0 < a.r; j0 += 8)
                                    tma_load_3d(gbase + (size_t)bq * BcBytes + (size_t)((s2 * a.r + j0) / 8) * 2048u, mB,
                                                &bcload[ps], j0, (a.G * it.gi + bq) * kTileM, e);
                            }
                        loaded = pseq;
                        if (pseq == 0) *s_bfirst = 1;
                    }
                    ok = mbar_wait(&bcload[ps], (uint32_t)((pseq / NP) & 1), abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const int groups = a.Kp / 8;
                    const int chunks = it.nb * groups * kTileM;      // 16-byte chunks: (block, column group, row)
                    // the first group with the eight epilogue warps (which
                    // have no accumulator to read yet), the others alone
                    const bool first = pseq == 0;
                    scale_bcat_chunks(gbase, chunks, groups, a.r, a.ns, s_e, s_g, tb, first ? 64 + 32 * kEpiWarps : 64);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (first) {
                        ok = mbar_wait(b0done, 0u, abort_flag);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                    }
                    if (lane == 0) mbar_arrive(&bcfull[ps]);
                }
                if (i + 1 < count) it.next(a.lins, a.n_lin);
            }
            // After an abort the last B loads may still be in flight.
            if (warp == 2 && lane == 0 && loaded >= 0)
                mbar_wait_drain(&bcload[loaded % NP], (uint32_t)((loaded / NP) & 1));
        }
    } else if (warp >= 4 && warp < 4 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        if (!kTB && count > 0) {
            // help the two builder warps scale the first group's B rows
            GroupTileIt it0;
            it0.init(a.lins, a.n_lin, t_begin, a.G);
            bool ok = mbar_wait(&bcload[0], 0u, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const int groups = a.Kp / 8;
                scale_bcat_chunks(sBcat, it0.nb * groups * kTileM, groups, a.r, a.ns, s_e, s_g,
                                  64 + (warp - 4) * 32 + lane, 64 + 32 * kEpiWarps);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b0done);
        }
        const int ew = warp - 4;
        const int q = warp & 3;
        const int h = ew >> 2;
        const int row = q * 32 + lane;
        GroupTileIt it;
        if (count > 0) it.init(a.lins, a.n_lin, t_begin, a.G);
        int64_t stored = 0;
        for (int64_t i = 0; i < count; ++i) {
            const int acc = (int)(i & 1);
            const int sw = (int)(i % a.SW);
            bool ok = mbar_wait(&accfull[acc], (uint32_t)((i >> 1) & 1), abort_flag);
            ok = ok && mbar_wait(&full[sw], (uint32_t)((i / a.SW) & 1), abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t va[32], vb[32];
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * kTileN + (uint32_t)h * 64u;
            tc_ld_x32(taddr, va);
            tc_ld_x32(taddr + 32u, vb);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            uint8_t* slice = sStage + (size_t)sw * a.stage_bytes + (size_t)h * kWBoxBytes + (size_t)q * 32 * 128;
            const uint32_t wrow = smem_u32(slice) + (uint32_t)lane * 128u;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t addr = wrow + ((uint32_t)(c ^ (row & 7)) << 4);
                const uint4 w = ld_shared_v4(addr);
                const uint32_t* dd = (c < 4) ? &va[c * 8] : &vb[(c - 4) * 8];
                uint4 o;
                o.x = add_bf16x2(w.x, dd[0], dd[1]);
                o.y = add_bf16x2(w.y, dd[2], dd[3]);
                o.z = add_bf16x2(w.z, dd[4], dd[5]);
                o.w = add_bf16x2(w.w, dd[6], dd[7]);
                st_shared_v4(addr, o);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const CUtensorMap* mO = a.maps + (size_t)it.l * kMapsPerLinear + kMapWoutStore;
                tma_store_2d(mO, slice, it.strip * kTileN + h * 64, it.rt() * kTileM + q * 32);
                bulk_commit_group();
                bulk_wait_group_read<1>();
                if (i > 0) mbar_arrive(&empty[(i - 1) % a.SW]);
            }
            stored = i + 1;
            if (i + 1 < count) it.next(a.lins, a.n_lin);
        }
        if (lane == 0) {
            bulk_wait_group<0>();
            if (stored > 0) mbar_arrive(&empty[(stored - 1) % a.SW]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.status, ADAFUSE_STATUS_TIMEOUT);
}

// ------------------------------------------------------------------ baseline

// One launch per linear; each thread produces 8 consecutive outputs of a row
// with CUDA-core FMAs straight from global memory.
__global__ void __launch_bounds__(128) merge_per_linear_kernel(LinDesc L, const int32_t* idx, const float* gate,
                                                                int32_t k, int32_t E, int32_t r, int32_t* status)
{
    __shared__ int s_e[kMaxSlots];
    __shared__ float s_g[kMaxSlots];
    if (threadIdx.x < k) {
        int e = idx[threadIdx.x];
        float g = gate[threadIdx.x];
        if (e < 0 || e >= E) {
            if (blockIdx.x == 0 && blockIdx.y == 0) atomicOr(status, ADAFUSE_STATUS_BAD_INDEX);
            e = -1;
            g = 0.f;
        }
        s_e[threadIdx.x] = e;
        s_g[threadIdx.x] = g;
    }
    __syncthreads();
    const int o = blockIdx.y;
    const int i0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (i0 >= L.d_in) return;
    const uint4 w = ld_global_nc_v4(L.W + (int64_t)o * L.d_in + i0);
    float acc[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                    bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
    for (int s = 0; s < k; ++s) {
        const int e = s_e[s];
        if (e < 0) continue;
        const float g = s_g[s];
        const uint16_t* Bo = L.B + (int64_t)e * L.b_es + (int64_t)o * r;
        const uint16_t* Ae = L.A + (int64_t)e * L.a_es + i0;
        for (int j = 0; j < r; ++j) {
            const float b = g * __uint_as_float((uint32_t)Bo[j] << 16);
            const uint4 av = ld_global_nc_v4(Ae + (int64_t)j * L.d_in);
            acc[0] += b * bf16lo(av.x); acc[1] += b * bf16hi(av.x);
            acc[2] += b * bf16lo(av.y); acc[3] += b * bf16hi(av.y);
            acc[4] += b * bf16lo(av.z); acc[5] += b * bf16hi(av.z);
            acc[6] += b * bf16lo(av.w); acc[7] += b * bf16hi(av.w);
        }
    }
    uint4 out;
    out.x = pack_bf16x2(acc[0], acc[1]);
    out.y = pack_bf16x2(acc[2], acc[3]);
    out.z = pack_bf16x2(acc[4], acc[5]);
    out.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(L.W_out + (int64_t)o * L.d_in + i0) = out;
}

}  // namespace

int launch_merge_fused(Plan* p, const int32_t* idx0, const float* gate0, const int32_t* idx1,
                       const float* gate1, int32_t k, int mode, cudaStream_t s)
{
    MergeArgs a{};
    a.lins = p->d_desc;
    a.maps = p->d_maps;
    a.idx0 = idx0; a.gate0 = gate0;
    a.idx1 = idx1 ? idx1 : idx0; a.gate1 = gate1 ? gate1 : gate0;
    a.status = p->d_status;
    a.total_tiles = p->merge_tiles;
    a.n_lin = p->n_lin;
    a.E = p->E; a.r = p->r; a.k = k;
    a.ns = mode == 1 ? 2 * k : k;
    a.Kp = ((a.ns * p->r + 15) / 16) * 16;
    a.mode = mode;
    if (a.ns > kMaxSlots || a.Kp > kMaxKr) return ADAFUSE_ERR_UNSUPPORTED;

    const uint32_t kSmemMax = 232448u;
    a.stall = (p->flags & ADAFUSE_PLAN_TEST_STALL) ? 1 : 0;
    a.box_rows = p->a_box_rows;
    if (a.Kp <= 128) {
        // Row-order kernel: W stages (up to four), a ring of A tiles, and the
        // Bcat of one or two groups of G row blocks.  Preference: W stages,
        // then the group size (less A traffic), then a second group slot (the
        // next group's Bcat built ahead), then A slots.  Groups of four or
        // eight only where a CTA walks enough tiles to amortise their builds.
        // Single-block groups (a plain row walk, every tile its own A tile)
        // only where they buy a W stage: at k*r = 128, G = 1 with four W
        // stages ran the 13B switch 17 % faster than G = 2 with three.
        //
        // From a contraction depth of 64 (K a multiple of 32) the Bcat of each
        // group lives in TMEM instead (Kp / 2 columns per row block beside the
        // two accumulators, at most 256 columns), so shared memory holds only
        // W stages and A tiles and a group can share each A tile among more
        // row blocks without giving up a W stage.  Only on long walks: at
        // Kp = 32 the shared-memory Bcat measured faster (7B merge 4.52 vs
        // 4.57 ms), and on a single layer the first TMA-loaded Bcat is ready
        // sooner than one built from global loads (k*r = 128: 34.8 vs 39.7 us).
        const uint32_t at = (uint32_t)a.Kp * 256u;
        const bool long_walk = p->merge_tiles >= 128 * (int64_t)p->num_sms;
        const bool tb = long_walk && a.Kp >= 64 && a.Kp % 32 == 0;
        const uint32_t bc = tb ? 0u : at;                    // smem per Bcat block
        // Up to four W stages; a fifth in the switch (in place) with the B rows
        // in TMEM, where it measured faster (13B switch 10.6 -> 10.2 ms, 7B
        // switch 5.05 -> 4.90 ms) while it slowed the 13B merge (8.87 -> 9.38).
        const int64_t sw_cap = (tb && a.mode == 1) ? 5 : 4;
        int SW = 0, NA = 0, NAR = 0, G = 0;
        for (int g : {8, 4, 2, 1}) {
            if (g >= 4 && !long_walk) continue;
            for (int np : {2, 1}) {
                if (tb && np * g * (a.Kp / 2) > 256) continue;
                for (int nar : {3, 2}) {
                    const int64_t room = (int64_t)kSmemMax - 2048 - (int64_t)np * g * bc - (int64_t)nar * at;
                    const int sw = room > 0 ? (int)std::min<int64_t>(sw_cap, room / kWTileBytes) : 0;
                    if (sw > SW) { SW = sw; NA = np * g; NAR = nar; G = g; }
                }
            }
        }
        if (SW >= 2) {
            a.SW = SW; a.SB = 0; a.NA = NA; a.NAR = NAR; a.G = G;
            a.stage_bytes = kWTileBytes;
            a.off_A = (uint32_t)SW * kWTileBytes;
            a.off_B = a.off_A + (uint32_t)NAR * at;
            a.off_bar = a.off_B + (uint32_t)NA * bc;
            const uint32_t smem = a.off_bar + 1024u + 1024u;
            const int grid = (int)std::min<int64_t>(p->num_sms, p->merge_tiles);
            p->last_launches = 1;
            if (tb) {
                if (cudaFuncSetAttribute(merge_rows_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem) != cudaSuccess)
                    return ADAFUSE_ERR_CUDA;
                return launch_pdl(merge_rows_kernel<true>, dim3(grid), dim3(kMergeThreadsTB), smem, s, a);
            }
            if (cudaFuncSetAttribute(merge_rows_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess)
                return ADAFUSE_ERR_CUDA;
            return launch_pdl(merge_rows_kernel<false>, dim3(grid), dim3(kMergeThreads), smem, s, a);
        }
    }
    const uint32_t BBytes = (uint32_t)a.Kp * 256u;
    const uint32_t ABytes = BBytes;                  // 227 KB opt-in per block
    const uint32_t extra = 1024u /*alignment*/ + 1024u /*barriers, slots*/;
    int NA = 2, SB = 2, SW = 0;
    auto fits = [&](int sw, int sb, int na) {
        return (uint64_t)sw * kWTileBytes + (uint64_t)sb * BBytes + (uint64_t)na * ABytes + extra <= kSmemMax;
    };
    // The epilogue releases a W stage one tile late (after the next tile's
    // store has been issued), so the W ring needs at least two stages.
    for (int sw = 6; sw >= 2 && SW == 0; --sw) if (fits(sw, SB, NA)) SW = sw;
    if (SW == 0) { NA = 1; SB = 2; for (int sw = 6; sw >= 2 && SW == 0; --sw) if (fits(sw, SB, NA)) SW = sw; }
    if (SW == 0) { NA = 1; SB = 1; for (int sw = 6; sw >= 2 && SW == 0; --sw) if (fits(sw, SB, NA)) SW = sw; }
    if (SW == 0) return ADAFUSE_ERR_UNSUPPORTED;
    a.SW = SW; a.SB = SB; a.NA = NA;
    a.off_B = (uint32_t)SW * kWTileBytes;
    a.off_A = a.off_B + (uint32_t)SB * BBytes;
    a.off_bar = a.off_A + (uint32_t)NA * ABytes;
    const uint32_t smem = a.off_bar + 1024u + 1024u;

    cudaError_t e = cudaFuncSetAttribute(merge_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
    const int grid = (int)std::min<int64_t>(p->num_sms, p->merge_tiles);
    p->last_launches = 1;
    return launch_pdl(merge_fused_kernel, dim3(grid), dim3(kMergeThreads), smem, s, a);
}

int launch_merge_per_linear(Plan* p, const int32_t* idx, const float* gate, int32_t k, cudaStream_t s)
{
    int launches = 0;
    for (int l = 0; l < p->n_lin; ++l) {
        const LinDesc& L = p->h_desc[l];
        dim3 grid((unsigned)((L.d_in + 8 * 128 - 1) / (8 * 128)), (unsigned)L.d_out);
        merge_per_linear_kernel<<<grid, 128, 0, s>>>(L, idx, gate, k, p->E, p->r, p->d_status);
        ++launches;
    }
    p->last_launches = launches;
    return cuda_err(cudaGetLastError());
}

}  // namespace af
