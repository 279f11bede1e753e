// Segmented-gather apply for mixed-adapter batches (unmerged form):
//   y_l = x_l W_l^T + sum_s g_s (x_l A_{e_s}^T) B_{e_s}^T     for every linear l.
//
// AdaFuse names the kernel "Segmented Gather Matrix Multiplication" (page pt
// section 2.B); the pages print no formula for the unmerged form, so it is the
// plain mixed-batch LoRA product above, per token with that token's top-k.
//
// Launches per call, independent of the number of layers:
//   1. segments  stable sort of the (token, slot) pairs by expert (segments.cu);
//                gives the U experts the batch uses, and clears the counters
//                that the later launches synchronise through;
// then, for plans with at least one apply unit per SM or more than 8 tokens:
//   2. shrink    (128-row tile of Acat, K-slice of a linear, token tile):
//                the used experts' stacked A rows times x_l^T on the tensor
//                cores, fp32 partials to the workspace;
//   3. finalize  per (linear, token): the K-slices added in order, the
//                token's gates applied, stored as a bf16 hi/lo pair
//                S_l[T, 2 * Kext] (hi and lo interleaved by groups of 32
//                columns);
//   4. apply     (linear, block of 128, 256 or 512 output rows, token tile):
//                D[rows x Npad] = W_block x^T (d_in/64 swizzled K chunks)
//                then + Bcat_block S^T (the used experts' B rows, gathered by
//                TMA, against both halves of S), all in one fp32 TMEM
//                accumulator, then y = bf16(D^T);
// and for smaller plans (a layer or a few, at most 8 tokens) the shrink units
// run inside the apply kernel instead (two launches): queued before the apply
// units, finalized by the warp that completes a 32-row slice last among its
// K-slices, and the apply units load their expand chunks once every slice of
// their linear's S is done (a bounded wait that, coming after all shrink
// units in the queue, never waits on work that has not started).  Below one
// unit per SM, units are split along K (a range of the base chunks and a
// range of the expand chunks each) and the last split of each 32-row slice
// adds the fp32 partials in split order.
// Every operand moves by TMA: W and the experts' A and B rows through the
// plan's tensor maps, x and S through per-call maps that the host builds (and
// caches by pointer set, T, k and workspace) before the launches.  W is streamed
// exactly once per token tile; the x and S tiles come from L2.  All launches
// use programmatic dependent launch: each kernel sets up its shared memory
// while the previous one runs and waits for it before touching what it wrote;
// the apply kernel also issues its first unit's first W and x loads before
// that wait (no launch of the call writes W or x).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace af {

namespace {

// ------------------------------------------------------------------ workspace

struct WsLayout {
    size_t off_offsets, off_used, off_perm, off_S, off_P, off_Yp, off_cnt, off_scnt, off_ready, total;
    int64_t n_zero;         // int32 counters from off_cnt on, cleared by the segment build
    int32_t Umax, Kext, Mt, Npad, n_tt;
    int32_t shape, tile;    // apply units of 128 << shape rows; tokens per tile
    int32_t ksg, total_ks;  // shrink K-slice width shrink_ks(ksg); slices over all linears
    int32_t nsplit;         // K-splits per apply unit
    bool fused;             // shrink units inside the apply kernel (small plans, T <= 32)
    int64_t n_grp;          // apply units (before splitting) over all token tiles
    int64_t n_su;           // shrink units per token tile: Mt x total K-slices
};

constexpr int kMaxSplit = 16;                     // K-splits per apply unit, at most

// Unit height for a batch of T tokens.  A taller unit issues more MMAs per x
// chunk it stages; its token tile (256 >> shape) must still cover T, or W is
// streamed once per extra tile.
int apply_shape(int64_t T) { return T <= 64 ? 2 : T <= 128 ? 1 : 0; }

int64_t token_tiles(int64_t T, int shape) { return (T + (256 >> shape) - 1) / (256 >> shape); }

WsLayout ws_layout(const Plan* p, int64_t T, int32_t k)
{
    WsLayout w{};
    const int64_t P = T * k;
    w.Umax = (int32_t)std::min<int64_t>(p->E, P);
    w.Kext = ((w.Umax * p->r + 63) / 64) * 64;
    w.Mt = (w.Umax * p->r + kTileM - 1) / kTileM;
    // Taller units only while they still give every SM two units or more;
    // below one unit per SM the units are split along K (base, then expand,
    // chunks), at least four chunks of the longest linear per split.
    w.shape = apply_shape(T);
    while (w.shape > 0 && p->apply_units[w.shape] * token_tiles(T, w.shape) < 2 * (int64_t)p->num_sms) --w.shape;
    w.tile = 256 >> w.shape;
    w.Npad = (int32_t)std::min<int64_t>(w.tile, ((T + 15) / 16) * 16);
    w.n_tt = (int32_t)token_tiles(T, w.shape);
    w.n_grp = p->apply_units[w.shape] * w.n_tt;
    // Split count: the fewest waves of equal units over the SMs, each split
    // charged a fixed 0.15 of a whole unit (pipeline fill, partial exchange).
    int max_kb = 1;
    for (const LinDesc& d : p->h_desc) max_kb = std::max(max_kb, (d.d_in + kChunkK - 1) / kChunkK);
    w.nsplit = 1;
    if (w.n_grp < p->num_sms) {
        double best = 1e30;
        for (int sp = 1; sp <= std::min(kMaxSplit, std::max(1, max_kb / 4)); ++sp) {
            const int64_t waves = (w.n_grp * sp + p->num_sms - 1) / p->num_sms;
            const double cost = (double)waves * (1.0 / sp + 0.15);
            if (cost < best - 1e-9) { best = cost; w.nsplit = sp; }
        }
    }
    // With fewer apply units than SMs and a few tokens, the shrink runs as
    // work units of the apply kernel, on the SMs the apply units leave free
    // and off the critical path; otherwise as a kernel of its own followed by
    // the finalize kernel (whose CTA per (linear, token) is the faster
    // finalize once a tile holds more than a few tokens).  Narrow shrink
    // slices only when the wide ones leave SMs without a unit.
    w.fused = w.n_grp < p->num_sms && T <= 8;
    w.ksg = (int64_t)w.Mt * p->total_ks[0] * token_tiles(T, w.shape) < p->num_sms ? 1 : 0;
    w.total_ks = p->total_ks[w.ksg];
    w.n_su = (int64_t)w.Mt * w.total_ks;
    auto up = [](size_t b) { return ((b + 255) / 256) * 256; };
    w.off_offsets = 0;
    w.off_used = 256;
    w.off_perm = 512;
    w.off_S = 512 + up((size_t)P * 4);
    w.off_P = w.off_S + up((size_t)p->n_lin * (size_t)T * (size_t)(2 * w.Kext) * 2);
    w.off_Yp = w.off_P + up((size_t)w.n_tt * (size_t)w.n_su * (size_t)w.Npad * kTileM * 4);
    const size_t rows_u = (size_t)kTileM << w.shape;
    const bool split = w.nsplit > 1;
    w.off_cnt = w.off_Yp + (split ? up((size_t)w.n_grp * w.nsplit * w.Npad * rows_u * 4) : 0);
    // Counters, all cleared by the segment build of every call: the apply
    // splits' per 32-row slice, the shrink's per (token tile, linear, Acat
    // tile, 32-row slice), and the finished S slices per (token tile, linear).
    const size_t n_cnt = split ? (size_t)w.n_grp * (rows_u / 32) : 0;
    w.off_scnt = w.off_cnt + n_cnt * 4;
    w.off_ready = w.off_scnt + (size_t)w.n_tt * p->n_lin * w.Mt * 4 * 4;
    const size_t end = w.off_ready + (size_t)w.n_tt * p->n_lin * 4;
    w.n_zero = (int64_t)((end - w.off_cnt) / 4);
    w.total = up(end);
    return w;
}

// Wait that ignores the abort flag (used to drain in-flight async work).
__device__ __forceinline__ bool mbar_wait_drain2(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

constexpr uint32_t kAChunkBytes = kTileM * kChunkK * 2;     // 16 KB: 128 rows x 64 cols bf16
// Pipeline stages of the shrink and apply kernels: as many as shared memory
// holds, up to 16 (small stages, e.g. one 16 KB W chunk and a few tokens of
// x, need many in flight per SM to cover the loaded memory latency).
constexpr int kMaxStages = 16;

// A shrink unit: Acat tile mq (rows mq*128 ..) against K-slice ks of linear
// l, columns [k0, k0 + nK * 64) of d_in.
struct ShrinkUnit {
    int l, mq, ks, k0, nK;
    __device__ void at(const LinDesc* lins, int n_lin, int total_ks, int ksg, int64_t u)
    {
        mq = (int)(u / total_ks);
        const int g = (int)(u - (int64_t)mq * total_ks);
        int lo = 0, hi = n_lin - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (__ldg(&lins[mid].ks_base[ksg]) <= g) lo = mid; else hi = mid - 1;
        }
        l = lo;
        ks = g - __ldg(&lins[l].ks_base[ksg]);
        const int width = shrink_ks(ksg);
        k0 = ks * width;
        const int k1 = min(__ldg(&lins[l].d_in), k0 + width);
        nK = (k1 - k0 + kChunkK - 1) / kChunkK;
    }
};

// ------------------------------------------------------------------ shrink
//
// S^T = Acat x^T for every linear, on the tensor cores: Acat stacks the A rows
// of the U used experts (U*r rows, gathered by TMA: boxes of 2-16 whole experts
// for runs of consecutive expert ids where r is a power of two, else boxes of
// up to 128 rows of one expert), x^T is the token tile.  Work units are
// (128-row tile of Acat, K-slice of a linear); each unit writes its fp32
// partial [Npad x 128] to the workspace.  Plans with at least one apply unit
// per SM run the shrink as this kernel of its own, followed by the finalize
// kernel (slices added in order, gates applied, rounded); smaller plans run
// the same units inside the apply kernel (below), finalized by the warp that
// completes a slice last.

struct ShrinkArgs {
    const LinDesc* lins;
    const CUtensorMap* maps;
    const CUtensorMap* xmaps;
    const int32_t* used;
    float* P;
    int32_t* status;
    int64_t n_su;
    int32_t n_lin, r, Npad, n_tt, total_ks, tile, ksg;
    int32_t ST, box_rows, run_max;
    uint32_t stage_bytes, off_bar, acc_stride, tmem_cols;
};

constexpr int kShrinkThreads = 192;

__global__ void __launch_bounds__(kShrinkThreads, 1) shrink_tc_kernel(const __grid_constant__ ShrinkArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + a.off_bar);
    uint64_t* empty = full + a.ST;
    uint64_t* accfull = empty + a.ST;
    uint64_t* accempty = accfull + 2;
    uint64_t* donebar = accempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(donebar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_used = reinterpret_cast<int*>(tmem_slot + 4);     // [1 + kMaxE]
    int* s_loads = s_used + 1 + kMaxE;                        // [kTileM / 8]: A loads of the current unit

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < a.ST; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 4); }
        mbar_init(donebar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int s = 0; s < a.ST; ++s)
        for (uint32_t o = threadIdx.x * 16; o < kAChunkBytes; o += kShrinkThreads * 16)
            st_shared_v4(smem_u32(base + (size_t)s * a.stage_bytes + o), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x <= kMaxE) s_used[threadIdx.x] = a.used[threadIdx.x];
    __syncthreads();
    const int rows = s_used[0] * a.r;          // live rows of Acat
    if (warp == 1) {
        tmem_alloc(tmem_slot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t total = a.n_su * a.n_tt;
    const int64_t u_begin = (int64_t)blockIdx.x * total / gridDim.x;
    const int64_t u_end = ((int64_t)blockIdx.x + 1) * total / gridDim.x;
    const uint32_t xbytes = (uint32_t)a.Npad * 128u;

    if (warp == 0) {
        if (lane == 0) {
            int64_t gc = 0, issued = 0;
            bool stop = false;
            for (int64_t ua = u_begin; ua < u_end && !stop; ++ua) {
                const int tt = (int)(ua / a.n_su);
                ShrinkUnit su;
                su.at(a.lins, a.n_lin, a.total_ks, a.ksg, ua - (int64_t)tt * a.n_su);
                if (su.mq * kTileM >= rows) continue;
                const CUtensorMap* mA = a.maps + (size_t)su.l * kMapsPerLinear + kMapA;
                const CUtensorMap* mX = a.xmaps + su.l;
                const int R = a.box_rows;               // A rows per box (divides r and 128)
                int ng = 0;
                for (int g = 0; g < kTileM / R; ++g) if (su.mq * kTileM + g * R < rows) ++ng;
                // One box per expert (R == r): a run of consecutive expert ids
                // is loaded in pieces of 2^i whole experts.  Entry: expert |
                // map << 8 | tile position << 16.
                int nload = 0;
                if (a.run_max > 1) {
                    const int q0 = su.mq * (kTileM / R), q1 = q0 + ng;
                    for (int q = q0; q < q1;) {
                        int e = s_used[1 + q], L = 1;
                        while (q + L < q1 && s_used[1 + q + L] == e + L) ++L;
                        while (L > 0) {
                            int D = 1, mi = -1;
                            while (2 * D <= L && 2 * D <= a.run_max) { D *= 2; ++mi; }
                            s_loads[nload++] = e | ((mi < 0 ? kMapA : kMapARun + mi) << 8) | ((q - q0) << 16);
                            q += D; e += D; L -= D;
                        }
                    }
                }
                for (int kc = 0; kc < su.nK; ++kc, ++gc) {
                    const int s = (int)(gc % a.ST);
                    if (!mbar_wait(&empty[s], (uint32_t)((gc / a.ST) & 1) ^ 1u, abort_flag)) { stop = true; break; }
                    uint8_t* dst = base + (size_t)s * a.stage_bytes;
                    const int col = su.k0 + kc * kChunkK;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(ng * R) * 128u + xbytes);
                    if (a.run_max > 1) {
                        for (int i = 0; i < nload; ++i) {
                            const int v = s_loads[i];
                            tma_load_3d(dst + (size_t)(v >> 16) * R * 128u,
                                        a.maps + (size_t)su.l * kMapsPerLinear + ((v >> 8) & 0xff), &full[s], col, 0,
                                        v & 0xff);
                        }
                    } else {
                        for (int g = 0; g < ng; ++g) {
                            const int c = su.mq * kTileM + g * R;
                            const int qq = c / a.r, j0 = c - qq * a.r;
                            tma_load_3d(dst + (size_t)g * R * 128u, mA, &full[s], col, j0, s_used[1 + qq]);
                        }
                    }
                    tma_load_2d(dst + kAChunkBytes, mX, &full[s], col, tt * a.tile);
                    issued = gc + 1;
                }
            }
            for (int64_t g = std::max<int64_t>(0, issued - a.ST); g < issued; ++g)
                mbar_wait_drain2(&full[g % a.ST], (uint32_t)((g / a.ST) & 1));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(kTileM, (uint32_t)a.Npad, 0u, 0u);
            int64_t gc = 0, uc = 0;
            bool stop = false;
            for (int64_t ua = u_begin; ua < u_end && !stop; ++ua) {
                const int tt = (int)(ua / a.n_su);
                ShrinkUnit su;
                su.at(a.lins, a.n_lin, a.total_ks, a.ksg, ua - (int64_t)tt * a.n_su);
                if (su.mq * kTileM >= rows) continue;
                const int acc = (int)(uc & 1);
                if (!mbar_wait(&accempty[acc], (uint32_t)((uc >> 1) & 1) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)acc * a.acc_stride;
                for (int kc = 0; kc < su.nK; ++kc, ++gc) {
                    const int s = (int)(gc % a.ST);
                    if (!mbar_wait(&full[s], (uint32_t)((gc / a.ST) & 1), abort_flag)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(base + (size_t)s * a.stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < kChunkK / 16; ++kk)
                        tc_mma_bf16(d, make_sdesc(aaddr + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128),
                                    make_sdesc(aaddr + kAChunkBytes + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128),
                                    idesc, (kc | kk) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                if (stop) break;
                tc_commit(&accfull[acc]);
                ++uc;
            }
            tc_commit(donebar);
            mbar_wait_drain2(donebar, 0);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        int64_t uc = 0;
        for (int64_t ua = u_begin; ua < u_end; ++ua) {
            const int tt = (int)(ua / a.n_su);
            const int64_t u = ua - (int64_t)tt * a.n_su;
            ShrinkUnit su;
            su.at(a.lins, a.n_lin, a.total_ks, a.ksg, u);
            if (su.mq * kTileM >= rows) continue;
            const int acc = (int)(uc & 1);
            bool ok = mbar_wait(&accfull[acc], (uint32_t)((uc >> 1) & 1), abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            float* Pu = a.P + ((int64_t)tt * a.n_su + u) * a.Npad * kTileM + q * 32 + lane;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * a.acc_stride;
            for (int c0 = 0; c0 < a.Npad; c0 += 32) {
                uint32_t v[32];
                if (a.Npad - c0 >= 32) {
                    tc_ld_x32(tbase + (uint32_t)c0, v);
                } else {
                    uint32_t h[16];
                    tc_ld_x16(tbase + (uint32_t)c0, h);
#pragma unroll
                    for (int i = 0; i < 16; ++i) { v[i] = h[i]; v[16 + i] = 0; }
                }
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (c0 + i < a.Npad) Pu[(int64_t)(c0 + i) * kTileM] = __uint_as_float(v[i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            ++uc;
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, a.tmem_cols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.status, ADAFUSE_STATUS_TIMEOUT);
}

// s = coef(t, c) * (sum over the K-slices of linear l of the partials), for
// c < U*r (zero for the padding columns up to Kext); coef(t, c) is the sum of
// token t's gates on expert used[1 + c/r] (zero if t did not pick it).  s is
// stored as two bf16 values, hi = bf16(s) and lo = bf16(s - hi), whose sum
// carries s to about 2^-17 relative: the expand multiplies both halves by the
// same B rows, so the LoRA term keeps close to fp32 precision even where it
// cancels most of the base product.  Row layout of S_l[t]: for each group of
// 32 columns, its 32 hi values then its 32 lo values, so that one 64-column
// box of S feeds both halves of an expand chunk.
__global__ void __launch_bounds__(128) shrink_finalize_kernel(const LinDesc* lins, const float* P, const int32_t* used,
                                                               const int32_t* idx, const float* gate, uint16_t* S,
                                                               int64_t T, int32_t k, int32_t r, int32_t Kext,
                                                               int32_t Npad, int32_t tile, int64_t n_su,
                                                               int32_t total_ks, int32_t ksg)
{
    griddep_wait();
    griddep_launch_dependents();
    __shared__ int s_used[kMaxE + 1];
    __shared__ int s_idx[kMaxSlots];
    __shared__ float s_gate[kMaxSlots];
    const int l = blockIdx.x;
    const int64_t t = blockIdx.y;
    if (threadIdx.x <= kMaxE) s_used[threadIdx.x] = used[threadIdx.x];
    if (threadIdx.x < k) { s_idx[threadIdx.x] = idx[t * k + threadIdx.x]; s_gate[threadIdx.x] = gate[t * k + threadIdx.x]; }
    __syncthreads();
    const int rows = s_used[0] * r;
    const int ks_base = __ldg(&lins[l].ks_base[ksg]), n_ks = __ldg(&lins[l].n_ks[ksg]);
    const int tt = (int)(t / tile), tl = (int)(t - (int64_t)tt * tile);
    uint16_t* Srow = S + ((int64_t)l * T + t) * (2 * Kext);
    for (int c = threadIdx.x; c < Kext; c += blockDim.x) {
        float v = 0.f;
        if (c < rows) {
            const int e = s_used[1 + c / r];
            float coef = 0.f;
            for (int s = 0; s < k; ++s) if (s_idx[s] == e) coef += s_gate[s];
            if (coef != 0.f) {
                const int mq = c / kTileM, cl = c - mq * kTileM;
                const float* p = P + (((int64_t)tt * n_su + (int64_t)mq * total_ks + ks_base) * Npad + tl) * kTileM + cl;
                // 8 K-slices of loads in flight; the sum still runs over them in order
                float sum = 0.f;
                for (int ks0 = 0; ks0 < n_ks; ks0 += 8) {
                    float t8[8];
#pragma unroll
                    for (int q2 = 0; q2 < 8; ++q2)
                        t8[q2] = ks0 + q2 < n_ks ? p[(int64_t)(ks0 + q2) * Npad * kTileM] : 0.f;
#pragma unroll
                    for (int q2 = 0; q2 < 8; ++q2)
                        if (ks0 + q2 < n_ks) sum += t8[q2];
                }
                v = coef * sum;
            }
        }
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const int o = 64 * (c >> 5) + (c & 31);              // [hi 32 | lo 32] per 32-column group
        Srow[o] = __bfloat16_as_ushort(hi);
        Srow[o + 32] = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(hi)));
    }
}

// ------------------------------------------------------------------ apply

struct ApplyArgs {
    const LinDesc* lins;
    const CUtensorMap* maps;        // plan maps (W, A, B) per linear
    const CUtensorMap* xmaps;       // per call: x_l maps [n_lin], then the shrink-output map
    void* const* y_ptrs;            // per call, device table: bf16 [T, d_out] (fp32 with y_f32)
    const int32_t* used;
    const int2* order;              // units (linear, row block), longest first
    int32_t* sched;                 // [0] next unit, [1] CTAs finished (both back to 0 at exit)
    int32_t* status;
    const int32_t* idx;             // [T, k] expert of each (token, slot)
    const float* gate;              // [T, k]
    uint16_t* S;                    // gated shrink, [n_lin][T][2 * Kext] bf16 hi/lo
    float* P;                       // shrink partials [n_tt][n_su][Npad][128] fp32
    int32_t* scnt;                  // [n_tt][n_lin][Mt][4] K-slices done per 32-row slice of an Acat tile
    int32_t* ready;                 // [n_tt][n_lin] finished 32-row slices of S
    int64_t T;
    int32_t n_lin, r, k, Npad, n_tt, n_units, Kext, tile, Mt;
    int32_t n_sh;                   // shrink units (n_tt * n_su), queued before the apply units
    int32_t n_su, total_ks, ksg;    // shrink units per token tile; K-slices over all linears; slice width
    int32_t box_rows, run_max;      // A-stack boxes: rows per box; most experts per load
    int32_t nsplit;                 // K-splits per unit (1: no split)
    int32_t bcols;                  // columns per B-row box of the expand: 8, 16 or 32
    int32_t stall;                  // test hook: CTA 0 withholds its first stage
    int32_t y_f32;                  // outputs are the fp32 accumulators (ADAFUSE_PLAN_Y_F32), not bf16
    float* Yp;                      // split partials [groups][nsplit][Npad][128 H] fp32
    int32_t* cnt;                   // [groups] splits finished (cleared by the segment build)
    int32_t ST;
    uint32_t stage_bytes, off_bar, acc_stride, tmem_cols;
};

// Writes one output row's values for up to 32 consecutive tokens: v[i] (fp32
// bits) goes to y[off + i * d_out] for i < min(n, t_left), rounded to bf16 or,
// with y_f32, as the fp32 value itself.  Lanes hold consecutive rows, so each
// store instruction of the warp covers 32 consecutive outputs of one token.
__device__ __forceinline__ void store_y_rows(void* y, int y_f32, int64_t off, int d_out, int n, int64_t t_left,
                                             const uint32_t (&v)[32])
{
    if (y_f32) {
        float* yp = static_cast<float*>(y) + off;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < n && i < t_left) yp[(int64_t)i * d_out] = __uint_as_float(v[i]);
    } else {
        uint16_t* yp = static_cast<uint16_t*>(y) + off;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < n && i < t_left) yp[(int64_t)i * d_out] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[i])));
    }
}

// Reads 32 accumulator columns [c0, c0 + 32) of this warp's TMEM lanes (16
// when only 16 remain below Npad; the rest read as zero).
__device__ __forceinline__ void tmem_cols32(uint32_t taddr, int remaining, uint32_t (&v)[32])
{
    if (remaining >= 32) {
        tc_ld_x32(taddr, v);
        tc_wait_ld();
    } else {
        uint32_t h[16];
        tc_ld_x16(taddr, h);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) { v[i] = h[i]; v[16 + i] = 0; }
    }
}

// A unit's share of the chunk list of its linear: nKb base chunks, then nKe
// expand chunks, split into nsplit contiguous ranges.
__device__ __forceinline__ void split_range(int n, int nsplit, int s, int& c0, int& c1)
{
    c0 = (int)((int64_t)s * n / nsplit);
    c1 = (int)((int64_t)(s + 1) * n / nsplit);
}

template <int H> struct ApplyShape {
    static constexpr int kEpiWarps = 4 * H;         // four per 128-row block
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
};
constexpr int kUnitRing = 4;

// Last CTA out puts the work counters back to zero for the next launch.
__device__ __forceinline__ void release_counters(int32_t* sched)
{
    __threadfence();
    if (atomicAdd(&sched[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&sched[0], 0);
        atomicExch(&sched[1], 0);
        __threadfence();
    }
}

// The finalize of one 32-row slice of an Acat tile (rows c = c_base + lane)
// for the tokens of token tile tt: the K-slices' fp32 partials added in slice
// order, times coef(t, c) = the sum of token t's gates on expert
// used[1 + c / r] (zero if t did not pick it; zero for c >= U * r), stored as
// hi = bf16(s) and lo = bf16(s - hi), whose sum carries s to about 2^-17
// relative: the expand multiplies both halves by the same B rows, so the LoRA
// term keeps close to fp32 precision even where it cancels most of the base
// product.  Row layout of S_l[t]: for each group of 32 columns, its 32 hi
// values then its 32 lo values, so that one 64-column box of S feeds both
// halves of an expand chunk.
__device__ __forceinline__ void finalize_slice(const ApplyArgs& a, const int* s_used, int l, int tt, int mq, int q,
                                               int lane)
{
    constexpr int kTok = 4;                                  // tokens per step: independent loads in flight
    const int rows = s_used[0] * a.r;
    const int c = mq * kTileM + q * 32 + lane;
    if (c >= a.Kext) return;
    const int e = c < rows ? s_used[1 + c / a.r] : -1;
    const int ks_base = __ldg(&a.lins[l].ks_base[a.ksg]), n_ks = __ldg(&a.lins[l].n_ks[a.ksg]);
    const float* p = a.P + (((int64_t)tt * a.n_su + (int64_t)mq * a.total_ks + ks_base) * a.Npad) * kTileM +
                     q * 32 + lane;
    const int64_t slice = (int64_t)a.Npad * kTileM;
    const int64_t t_left = a.T - (int64_t)tt * a.tile;
    const int n_tok = t_left < a.Npad ? (int)t_left : a.Npad;
    for (int tl0 = 0; tl0 < n_tok; tl0 += kTok) {
        float coef[kTok], sum[kTok];
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            coef[j] = 0.f;
            sum[j] = 0.f;
            const int64_t t = (int64_t)tt * a.tile + tl0 + j;
            if (e >= 0 && tl0 + j < n_tok)
                for (int s = 0; s < a.k; ++s)
                    if (__ldg(&a.idx[t * a.k + s]) == e) coef[j] += __ldg(&a.gate[t * a.k + s]);
        }
        // 8 K-slices x kTok tokens of partials in flight per L2 round trip;
        // each sum still runs over the slices in order
        for (int ks0 = 0; ks0 < n_ks; ks0 += 8) {
            float v[8][kTok];
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2)
#pragma unroll
                for (int j = 0; j < kTok; ++j)
                    v[q2][j] = (ks0 + q2 < n_ks && coef[j] != 0.f)
                                   ? __ldcg(p + (int64_t)(ks0 + q2) * slice + (int64_t)(tl0 + j) * kTileM)
                                   : 0.f;
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2)
                if (ks0 + q2 < n_ks) {
#pragma unroll
                    for (int j = 0; j < kTok; ++j) sum[j] += v[q2][j];
                }
        }
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            if (tl0 + j >= n_tok) break;
            const int64_t t = (int64_t)tt * a.tile + tl0 + j;
            const float v = coef[j] * sum[j];
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            uint16_t* Srow = a.S + ((int64_t)l * a.T + t) * (2 * a.Kext);
            const int o = 64 * (c >> 5) + (c & 31);          // [hi 32 | lo 32] per 32-column group
            Srow[o] = __bfloat16_as_ushort(hi);
            Srow[o + 32] = __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(hi)));
        }
    }
}

// Warp roles: 0 = TMA producer and work fetcher, 1 = TMEM owner and MMA
// issuer, 2.. = epilogue (four warps per 128-row block).  Units are fetched
// from a global counter -- the shrink units first, then the apply units,
// longest first -- so SMs that stream faster take more of them; the producer
// passes each unit id to the other roles through a small ring in shared
// memory.  Stage s holds H 128 x 64 A-operand chunks (W rows, the used
// experts' B rows, or for a shrink unit their A rows in chunk 0) and one
// Npad x 64 B-operand chunk (x rows, or shrink-output rows) that the MMAs
// share, all K-major; W, A and x use the 128-byte swizzle, B rows the layouts
// of their boxes.  Block h of an apply unit accumulates in TMEM columns
// [h*Npad, (h+1)*Npad) of the unit's accumulator; a shrink unit uses block 0.
template <int H, bool kFused>
__global__ void __launch_bounds__(ApplyShape<H>::kThreads, 1) apply_fused_kernel(const __grid_constant__ ApplyArgs a)
{
    constexpr int kApplyEpiWarps = ApplyShape<H>::kEpiWarps;
    constexpr int kApplyThreads = ApplyShape<H>::kThreads;
    constexpr int kApplyRows = kTileM * H;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + a.off_bar);
    uint64_t* empty = full + a.ST;
    uint64_t* accfull = empty + a.ST;
    uint64_t* accempty = accfull + 2;
    uint64_t* ufull = accempty + 2;
    uint64_t* uempty = ufull + kUnitRing;
    uint64_t* donebar = uempty + kUnitRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(donebar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_unit = reinterpret_cast<int*>(tmem_slot + 4);       // [kUnitRing]
    int* s_used = s_unit + kUnitRing;                           // [1 + kMaxE]
    int* s_loads = s_used + 1 + kMaxE;                          // [kTileM / 8]: A loads of a shrink chunk
    int* s_first = s_loads + kTileM / 8;                        // [2]: first unit, its stages loaded early

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = a.n_sh + a.n_units * a.n_tt * a.nsplit;
    const uint32_t xbytes = (uint32_t)a.Npad * 128u;
    if (threadIdx.x == 0) {
        for (int i = 0; i < a.ST; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], kApplyEpiWarps); }
        for (int i = 0; i < kUnitRing; ++i) { mbar_init(&ufull[i], 1); mbar_init(&uempty[i], 1 + kApplyEpiWarps); }
        mbar_init(donebar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // The CTA's first unit, and for an apply unit the W and x of its first
        // stages, before the wait: no launch of the call writes W or x, the
        // base chunk range does not depend on the selection, and the kernel
        // this one follows has itself waited for every earlier launch of the
        // stream (whose last CTA also put the work counter back to zero).
        int u = atomicAdd(&a.sched[0], 1);
        if (u >= total) u = -1;
        int ne = 0;
        if (u >= a.n_sh) {
            const int ua = u - a.n_sh;
            const int g = ua / a.nsplit, sp = ua - g * a.nsplit;
            const int tt = g / a.n_units;
            const int2 lm = a.order[g - tt * a.n_units];
            const int nKb = (__ldg(&a.lins[lm.x].d_in) + kChunkK - 1) / kChunkK;
            int b0, b1;
            split_range(nKb, a.nsplit, sp, b0, b1);
            // at most four stages: a whole ring from every CTA at once queues
            // the shrink's and finalize's loads behind it (one 4096 x 4096
            // layer: 29.7 -> 27.8 us at T = 1, 37.0 -> 36.0 us at T = 16)
            ne = min(min(4, a.ST), b1 - b0);
            const CUtensorMap* mW = a.maps + (size_t)lm.x * kMapsPerLinear + kMapW;
            for (int i = 0; i < ne; ++i) {
                if (a.stall && blockIdx.x == 0 && i == 0) continue;      // test hook (below)
                uint8_t* dst = base + (size_t)i * a.stage_bytes;
                mbar_arrive_expect_tx(&full[i], kAChunkBytes * H + xbytes);
                for (int hh = 0; hh < H; ++hh)
                    tma_load_2d(dst + hh * kAChunkBytes, mW, &full[i], (b0 + i) * kChunkK, lm.y * kApplyRows + hh * kTileM);
                tma_load_2d(dst + kAChunkBytes * H, a.xmaps + lm.x, &full[i], (b0 + i) * kChunkK, tt * a.tile);
            }
        }
        s_first[0] = u;
        s_first[1] = ne;
    }
    __syncthreads();
    // Zero the A regions the early loads leave alone: expert chunks load only
    // the 8-column groups they use (a stage that held W keeps finite values).
    for (int s = s_first[1]; s < a.ST; ++s)
        for (uint32_t o = threadIdx.x * 16; o < kAChunkBytes * H; o += kApplyThreads * 16)
            st_shared_v4(smem_u32(base + (size_t)s * a.stage_bytes + o), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x <= kMaxE) s_used[threadIdx.x] = a.used[threadIdx.x];
    __syncthreads();
    const int U = s_used[0];
    const int rows_live = U * a.r;                          // live rows of Acat
    const int nKe = (rows_live + 31) / 32;                  // expand chunks: 32 columns of Bcat each
    const int ready_target = ((rows_live + kTileM - 1) / kTileM) * 4;   // 32-row S slices per linear

    if (warp == 1) {
        tmem_alloc(tmem_slot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int64_t gc = 0, issued = 0;
            const CUtensorMap* mS = a.xmaps + a.n_lin;
            bool stop = false;
            for (int ui = 0; !stop; ++ui) {
                const int j = ui & (kUnitRing - 1);
                if (!mbar_wait(&uempty[j], (uint32_t)((ui / kUnitRing) & 1) ^ 1u, abort_flag)) break;
                int u = ui == 0 ? s_first[0] : atomicAdd(&a.sched[0], 1);
                if (u >= total) u = -1;
                s_unit[j] = u;
                mbar_arrive(&ufull[j]);
                if (u < 0) break;
                if (kFused && u < a.n_sh) {
                    // shrink unit: the live A rows of Acat tile mq (boxes of
                    // whole experts, runs of consecutive expert ids in one
                    // load where r allows) and the x chunk, per 64 columns
                    const int tt = u / a.n_su;
                    ShrinkUnit su;
                    su.at(a.lins, a.n_lin, a.total_ks, a.ksg, u - (int64_t)tt * a.n_su);
                    if (su.mq * kTileM >= rows_live) continue;
                    const CUtensorMap* mA = a.maps + (size_t)su.l * kMapsPerLinear + kMapA;
                    const CUtensorMap* mX = a.xmaps + su.l;
                    const int R = a.box_rows;               // A rows per box (divides r and 128)
                    int ng = 0;
                    for (int g = 0; g < kTileM / R; ++g) if (su.mq * kTileM + g * R < rows_live) ++ng;
                    // entry: expert | map << 8 | tile position << 16
                    int nload = 0;
                    if (a.run_max > 1) {
                        const int q0 = su.mq * (kTileM / R), q1 = q0 + ng;
                        for (int q = q0; q < q1;) {
                            int e = s_used[1 + q], L = 1;
                            while (q + L < q1 && s_used[1 + q + L] == e + L) ++L;
                            while (L > 0) {
                                int D = 1, mi = -1;
                                while (2 * D <= L && 2 * D <= a.run_max) { D *= 2; ++mi; }
                                s_loads[nload++] = e | ((mi < 0 ? kMapA : kMapARun + mi) << 8) | ((q - q0) << 16);
                                q += D; e += D; L -= D;
                            }
                        }
                    }
                    for (int kc = 0; kc < su.nK; ++kc, ++gc) {
                        const int s = (int)(gc % a.ST);
                        if (!mbar_wait(&empty[s], (uint32_t)((gc / a.ST) & 1) ^ 1u, abort_flag)) { stop = true; break; }
                        uint8_t* dst = base + (size_t)s * a.stage_bytes;
                        const int col = su.k0 + kc * kChunkK;
                        if (a.stall && blockIdx.x == 0 && gc == 0) {
                            // test hook: CTA 0 never loads its first stage
                        } else {
                            mbar_arrive_expect_tx(&full[s], (uint32_t)(ng * R) * 128u + xbytes);
                            if (a.run_max > 1) {
                                for (int i = 0; i < nload; ++i) {
                                    const int v = s_loads[i];
                                    tma_load_3d(dst + (size_t)(v >> 16) * R * 128u,
                                                a.maps + (size_t)su.l * kMapsPerLinear + ((v >> 8) & 0xff), &full[s],
                                                col, 0, v & 0xff);
                                }
                            } else {
                                for (int g = 0; g < ng; ++g) {
                                    const int c = su.mq * kTileM + g * R;
                                    const int qq = c / a.r, j0 = c - qq * a.r;
                                    tma_load_3d(dst + (size_t)g * R * 128u, mA, &full[s], col, j0, s_used[1 + qq]);
                                }
                            }
                            tma_load_2d(dst + kAChunkBytes * H, mX, &full[s], col, tt * a.tile);
                            issued = gc + 1;
                        }
                    }
                    continue;
                }
                const int ua = u - a.n_sh;
                const int g = ua / a.nsplit, sp = ua - g * a.nsplit;
                const int tt = g / a.n_units;
                const int2 lm = a.order[g - tt * a.n_units];
                const int l = lm.x;
                const int nKb = (__ldg(&a.lins[l].d_in) + kChunkK - 1) / kChunkK;
                // the split's base chunks, then its share of the expand chunks
                int b0, b1, e0, e1;
                split_range(nKb, a.nsplit, sp, b0, b1);
                split_range(nKe, a.nsplit, sp, e0, e1);
                const int nb = b1 - b0, nc = nb + (e1 - e0);
                const int n_early = ui == 0 ? s_first[1] : 0;
                const int m0 = lm.y * kApplyRows;
                const int t0 = tt * a.tile;
                const CUtensorMap* mW = a.maps + (size_t)l * kMapsPerLinear + kMapW;
                const CUtensorMap* mB = a.maps + (size_t)l * kMapsPerLinear + kMapB;
                const CUtensorMap* mB16 = a.maps + (size_t)l * kMapsPerLinear + kMapB16;
                const CUtensorMap* mB32 = a.maps + (size_t)l * kMapsPerLinear + kMapB32;
                const CUtensorMap* mX = a.xmaps + l;
                bool s_ready = false;
                for (int jc = 0; jc < nc; ++jc, ++gc) {
                    const int kc = jc < nb ? b0 + jc : nKb + e0 + (jc - nb);
                    if (jc < n_early) {                 // loaded before the wait
                        if (!(a.stall && blockIdx.x == 0 && gc == 0)) issued = gc + 1;
                        continue;
                    }
                    const int s = (int)(gc % a.ST);
                    if (kFused && kc >= nKb && !s_ready) {
                        // S of this linear and token tile: every 32-row slice
                        // finalized (released by the finalizing warps)
                        const int* rp = a.ready + (int64_t)tt * a.n_lin + l;
                        const uint64_t tw = globaltimer_ns();
                        while (ld_acquire_gpu(rp) < ready_target) {
                            if (*abort_flag || globaltimer_ns() - tw > kWaitLimitNs) { *abort_flag = 1; stop = true; break; }
                            __nanosleep(64);
                        }
                        if (stop) break;
                        fence_proxy_async_global();
                        s_ready = true;
                    }
                    if (!mbar_wait(&empty[s], (uint32_t)((gc / a.ST) & 1) ^ 1u, abort_flag)) { stop = true; break; }
                    uint8_t* dst = base + (size_t)s * a.stage_bytes;
                    if (a.stall && blockIdx.x == 0 && gc == 0) {
                        // test hook: CTA 0 never loads its first stage, so the
                        // MMA warp's wait on it runs out
                    } else if (kc < nKb) {
                        mbar_arrive_expect_tx(&full[s], kAChunkBytes * H + xbytes);
                        for (int hh = 0; hh < H; ++hh)
                            tma_load_2d(dst + hh * kAChunkBytes, mW, &full[s], kc * kChunkK, m0 + hh * kTileM);
                        tma_load_2d(dst + kAChunkBytes * H, mX, &full[s], kc * kChunkK, t0);
                        issued = gc + 1;
                    } else {
                        // expand: 32 columns of Bcat (the used experts' B
                        // rows) against the hi and the lo half of S for
                        // those columns, which sit side by side in one
                        // 64-column box of S; B rows in boxes of bcols
                        // columns (one expert each: bcols divides r), at
                        // bcols * 256 bytes per box
                        const int ke = kc - nKb;
                        const int col0 = ke * 32;
                        const int bc = a.bcols;
                        const CUtensorMap* mBx = bc == 32 ? mB32 : bc == 16 ? mB16 : mB;
                        int ng = 0;
                        for (int gg = 0; gg < 32 / bc; ++gg) if (col0 + gg * bc < rows_live) ++ng;
                        mbar_arrive_expect_tx(&full[s], (uint32_t)(ng * H * bc) * 256u + xbytes);
                        for (int hh = 0; hh < H; ++hh)
                            for (int gg = 0; gg < ng; ++gg) {
                                const int c = col0 + gg * bc;
                                const int qq = c / a.r, j0 = c - qq * a.r;
                                tma_load_3d(dst + hh * kAChunkBytes + (size_t)gg * bc * 256u, mBx, &full[s], j0,
                                            m0 + hh * kTileM, s_used[1 + qq]);
                            }
                        tma_load_3d(dst + kAChunkBytes * H, mS, &full[s], 2 * col0, t0, l);
                        issued = gc + 1;
                    }
                }
            }
            // Drain the TMA loads still in flight before the CTA may exit.
            for (int64_t g = std::max<int64_t>(0, issued - a.ST); g < issued; ++g)
                mbar_wait_drain2(&full[g % a.ST], (uint32_t)((g / a.ST) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(kTileM, (uint32_t)a.Npad, 0u, 0u);
            const int bmode = a.bcols == 32 ? 2 : a.bcols == 16 ? 1 : 0;
            int64_t gc = 0;
            bool stop = false;
            for (int ui = 0; !stop; ++ui) {
                const int j = ui & (kUnitRing - 1);
                if (!mbar_wait(&ufull[j], (uint32_t)((ui / kUnitRing) & 1), abort_flag)) break;
                const int u = s_unit[j];
                mbar_arrive(&uempty[j]);
                if (u < 0) break;
                int c0 = 0, c1 = 0, nKb = 0, b0 = 0, b1 = 0, e0 = 0, e1 = 0;
                const bool shrink = kFused && u < a.n_sh;
                if (shrink) {
                    const int tt = u / a.n_su;
                    ShrinkUnit su;
                    su.at(a.lins, a.n_lin, a.total_ks, a.ksg, u - (int64_t)tt * a.n_su);
                    if (su.mq * kTileM < rows_live) c1 = su.nK;          // dead tiles: an empty accumulator pass
                } else {
                    const int ua = u - a.n_sh;
                    const int g = ua / a.nsplit, sp = ua - g * a.nsplit;
                    const int l = a.order[g % a.n_units].x;
                    nKb = (__ldg(&a.lins[l].d_in) + kChunkK - 1) / kChunkK;
                    split_range(nKb, a.nsplit, sp, b0, b1);
                    split_range(nKe, a.nsplit, sp, e0, e1);
                    c1 = (b1 - b0) + (e1 - e0);
                }
                const int acc = ui & 1;
                if (!mbar_wait(&accempty[acc], (uint32_t)((ui >> 1) & 1) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)acc * a.acc_stride;
                for (int jc = c0; jc < c1; ++jc, ++gc) {
                    // shrink: chunk jc of the K-slice; apply: the split's base
                    // chunks, then its expand chunks
                    const int kc = shrink ? jc : jc < b1 - b0 ? b0 + jc : nKb + e0 + (jc - (b1 - b0));
                    const int s = (int)(gc % a.ST);
                    if (!mbar_wait(&full[s], (uint32_t)((gc / a.ST) & 1), abort_flag)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t abase = smem_u32(base + (size_t)s * a.stage_bytes);
                    const uint32_t baddr = abase + kAChunkBytes * H;
                    if (shrink) {
#pragma unroll
                        for (int kk = 0; kk < kChunkK / 16; ++kk)
                            tc_mma_bf16(d, make_sdesc(abase + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128),
                                        make_sdesc(baddr + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128), idesc,
                                        (jc != c0 || kk) ? 1u : 0u);
                        tc_commit(&empty[s]);
                        continue;
                    }
#pragma unroll
                    for (int hh = 0; hh < H; ++hh) {
                        const uint32_t aaddr = abase + hh * kAChunkBytes;
                        const uint32_t d_h = d + (uint32_t)(hh * a.Npad);
                        if (kc < nKb) {
#pragma unroll
                            for (int kk = 0; kk < kChunkK / 16; ++kk)
                                tc_mma_bf16(d_h, make_sdesc(aaddr + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128),
                                            make_sdesc(baddr + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128), idesc,
                                            (jc != c0 || kk) ? 1u : 0u);
                        } else {
                            // K steps 0-1 of the S chunk hold the hi half, 2-3 the
                            // lo half; both multiply the same 32 Bcat columns,
                            // whose 16-column K steps sit in: two 8-column
                            // core-matrix groups (no swizzle), one 16-column
                            // box (32-byte swizzle) or half of a 32-column box
                            // (64-byte swizzle)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t k2 = (uint32_t)(kk & 1);
                                const uint64_t adesc =
                                    bmode == 0 ? make_sdesc(aaddr + k2 * 4096u, 2048u, 128u, kLayoutNone)
                                    : bmode == 1 ? make_sdesc(aaddr + k2 * 4096u, 16u, 256u, kLayoutSw32)
                                                 : make_sdesc(aaddr + k2 * 32u, 16u, 512u, kLayoutSw64);
                                tc_mma_bf16(d_h, adesc, make_sdesc(baddr + (uint32_t)kk * 32u, 16u, 1024u, kLayoutSw128),
                                            idesc, (jc != c0 || kk) ? 1u : 0u);
                            }
                        }
                    }
                    tc_commit(&empty[s]);
                }
                if (stop) break;
                tc_commit(&accfull[acc]);
            }
            tc_commit(donebar);
            mbar_wait_drain2(donebar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Warp (hh, q) owns rows [hh*128 + q*32, +32) of an apply unit.
        // Without a K split it rounds its accumulator rows straight into y.
        // With one it stores them as an fp32 partial; the warp that finishes
        // its rows last among the unit's splits adds the partials in split
        // order (so the result does not depend on which split ends last) and
        // writes y.  For a shrink unit the warps of block 0 store their 32
        // Acat rows' partial, and the last of a slice's K-slices finalizes it.
        const int q = warp & 3;        // TMEM lane quarter: warps 2,3,4,5 -> 2,3,0,1
        const int hh = (warp - 2) >> 2;                        // which 128-row block
        const int rin = hh * kTileM + q * 32 + lane;           // row within the unit
        for (int ui = 0;; ++ui) {
            const int j = ui & (kUnitRing - 1);
            bool ok = mbar_wait(&ufull[j], (uint32_t)((ui / kUnitRing) & 1), abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int u = s_unit[j];
            __syncwarp();
            if (lane == 0) mbar_arrive(&uempty[j]);
            if (u < 0) break;
            const int acc = ui & 1;
            ok = mbar_wait(&accfull[acc], (uint32_t)((ui >> 1) & 1), abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * a.acc_stride;
            if (kFused && u < a.n_sh) {
                const int tt = u / a.n_su;
                const int64_t ul = u - (int64_t)tt * a.n_su;
                ShrinkUnit su;
                su.at(a.lins, a.n_lin, a.total_ks, a.ksg, ul);
                const bool mine = hh == 0 && su.mq * kTileM < rows_live;
                if (mine) {
                    float* Pu = a.P + ((int64_t)tt * a.n_su + ul) * a.Npad * kTileM + q * 32 + lane;
                    for (int c0 = 0; c0 < a.Npad; c0 += 32) {
                        uint32_t v[32];
                        tmem_cols32(tacc + (uint32_t)c0, a.Npad - c0, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c0 + i < a.Npad) Pu[(int64_t)(c0 + i) * kTileM] = __uint_as_float(v[i]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[acc]);
                if (mine) {
                    __threadfence();
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) {
                        const int n_ks = __ldg(&a.lins[su.l].n_ks[a.ksg]);
                        int32_t* cp = a.scnt + (((int64_t)tt * a.n_lin + su.l) * a.Mt + su.mq) * 4 + q;
                        last = atomicAdd(cp, 1) == n_ks - 1;
                    }
                    last = __shfl_sync(0xffffffffu, last, 0);
                    if (last) {
                        __threadfence();
                        finalize_slice(a, s_used, su.l, tt, su.mq, q, lane);
                        fence_proxy_async_global();       // S is read by TMA in other CTAs
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) atomicAdd(a.ready + (int64_t)tt * a.n_lin + su.l, 1);
                    }
                }
                continue;
            }
            const int ua = u - a.n_sh;
            const int g = ua / a.nsplit, sp = ua - g * a.nsplit;
            const int tt = g / a.n_units;
            const int2 lm = a.order[g - tt * a.n_units];
            const int d_out = __ldg(&a.lins[lm.x].d_out);
            void* y = a.y_ptrs[lm.x];
            const int64_t T = a.T;
            const int row = lm.y * kApplyRows + rin;
            const int64_t tb = (int64_t)tt * a.tile;
            const uint32_t tbase = tacc + (uint32_t)(hh * a.Npad);
            int kc0 = 0, kc1 = 1;                              // chunks of the split: none means a zero share
            if (a.nsplit > 1) {
                const int nKb = (__ldg(&a.lins[lm.x].d_in) + kChunkK - 1) / kChunkK;
                int b0, b1, e0, e1;
                split_range(nKb, a.nsplit, sp, b0, b1);
                split_range(nKe, a.nsplit, sp, e0, e1);
                kc1 = (b1 - b0) + (e1 - e0);
            }
            float* part = a.Yp + ((int64_t)ua * a.Npad) * kApplyRows + rin;
            const int n_tok = (int)min((int64_t)a.Npad, T - tb);     // the tile's tokens, without padding
            for (int c0 = 0; c0 < n_tok; c0 += 32) {
                uint32_t v[32];
                if (kc0 == kc1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0;       // empty split: its share is zero
                } else {
                    tmem_cols32(tbase + (uint32_t)c0, a.Npad - c0, v);
                }
                if (a.nsplit > 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c0 + i < n_tok) part[(int64_t)(c0 + i) * kApplyRows] = __uint_as_float(v[i]);
                } else if (row < d_out) {
                    store_y_rows(y, a.y_f32, (tb + c0) * d_out + row, d_out, n_tok - c0, n_tok - c0, v);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            // Units split along K only at H = 1 (fewer units than SMs).
            if (H == 1 && a.nsplit > 1) {
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0)
                    last = atomicAdd(&a.cnt[(int64_t)g * kApplyEpiWarps + (warp - 2)], 1) == a.nsplit - 1;
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    const float* p0 = a.Yp + ((int64_t)g * a.nsplit * a.Npad) * kApplyRows + rin;
                    for (int c0 = 0; c0 < n_tok; c0 += 16) {
                        // 16 tokens x 4 splits of loads in flight (one L2
                        // round trip per 4 splits, not per split); each sum
                        // still runs over the splits in order
                        float v[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = 0.f;
                        for (int s0 = 0; s0 < a.nsplit; s0 += 4) {
                            float t[4][16];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    t[j][i] = (s0 + j < a.nsplit && c0 + i < n_tok)
                                                  ? __ldcg(p0 + ((int64_t)(s0 + j) * a.Npad + c0 + i) * kApplyRows)
                                                  : 0.f;
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                if (s0 + j < a.nsplit) {
#pragma unroll
                                    for (int i = 0; i < 16; ++i) v[i] += t[j][i];
                                }
                        }
                        if (row < d_out) {
                            const int64_t off = (tb + c0) * d_out + row;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                if (c0 + i >= n_tok) break;
                                if (a.y_f32)
                                    static_cast<float*>(y)[off + (int64_t)i * d_out] = v[i];
                                else
                                    static_cast<uint16_t*>(y)[off + (int64_t)i * d_out] =
                                        __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
                            }
                        }
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, a.tmem_cols);
    }
    if (threadIdx.x == 0) {
        if (*abort_flag) atomicOr(a.status, ADAFUSE_STATUS_TIMEOUT);
        release_counters(a.sched);
    }
}

bool encode_tile_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                     const cuuint32_t* box)
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {     // resolved once, thread-safe
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// The two launches of one apply call: the segment build (which also clears
// the call's counters), then the fused shrink + apply kernel.  `xmaps` holds
// the call's x maps and then the shrink-output map, `yp` is the device table
// of output pointers and `wsb` the workspace laid out by `w`.
template <int H, bool kFused>
int launch_apply_fused(const ApplyArgs& a, uint32_t smem, int grid, cudaStream_t s)
{
    if (cudaFuncSetAttribute(apply_fused_kernel<H, kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return ADAFUSE_ERR_CUDA;
    return launch_pdl(apply_fused_kernel<H, kFused>, dim3(grid), dim3(ApplyShape<H>::kThreads), smem, s, a);
}

int launch_apply_kernels(Plan* p, const WsLayout& w, uint8_t* wsb, const CUtensorMap* xmaps, void* const* yp,
                         const int32_t* idx, const float* gate, int64_t T, int32_t k, cudaStream_t s)
{
    int32_t* offsets = reinterpret_cast<int32_t*>(wsb + w.off_offsets);
    int32_t* used = reinterpret_cast<int32_t*>(wsb + w.off_used);
    int32_t* perm = reinterpret_cast<int32_t*>(wsb + w.off_perm);
    const int32_t Npad = w.Npad;
    const int H = 1 << w.shape;
    const uint32_t kSmemMax = 232448u;

    int rc = launch_segments(idx, T, k, p->E, offsets, perm, used, p->d_status, s,
                             reinterpret_cast<int32_t*>(wsb + w.off_cnt), w.n_zero);
    if (rc != ADAFUSE_OK) return rc;

    if (!w.fused) {
        // The shrink as a kernel of its own, then the finalize.
        uint32_t accs = 32;
        while (accs < (uint32_t)Npad) accs <<= 1;
        const uint32_t stage_bytes = kAChunkBytes + (uint32_t)Npad * 128u;
        const int ST = std::min(kMaxStages, (int)((kSmemMax - 2048u) / stage_bytes));
        if (ST < 2 || 2 * accs > 512) return ADAFUSE_ERR_UNSUPPORTED;
        const uint32_t smem = (uint32_t)ST * stage_bytes + 1024u + 1024u;
        ShrinkArgs sa{};
        sa.lins = p->d_desc;
        sa.maps = p->d_maps;
        sa.xmaps = xmaps;
        sa.used = used;
        sa.P = reinterpret_cast<float*>(wsb + w.off_P);
        sa.status = p->d_status;
        sa.n_su = w.n_su;
        sa.n_lin = p->n_lin;
        sa.r = p->r;
        sa.Npad = Npad;
        sa.n_tt = w.n_tt;
        sa.total_ks = w.total_ks;
        sa.ksg = w.ksg;
        sa.tile = w.tile;
        sa.ST = ST;
        sa.box_rows = p->a_box_rows;
        sa.run_max = p->a_run_max;
        sa.stage_bytes = stage_bytes;
        sa.off_bar = (uint32_t)ST * stage_bytes;
        sa.acc_stride = accs;
        sa.tmem_cols = 2 * accs;
        if (cudaFuncSetAttribute(shrink_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return ADAFUSE_ERR_CUDA;
        rc = launch_pdl(shrink_tc_kernel, dim3((unsigned)std::min<int64_t>(p->num_sms, w.n_su * w.n_tt)),
                        dim3(kShrinkThreads), smem, s, sa);
        if (rc != ADAFUSE_OK) return rc;
        rc = launch_pdl(shrink_finalize_kernel, dim3((unsigned)p->n_lin, (unsigned)T), dim3(128), 0, s,
                        (const LinDesc*)p->d_desc, (const float*)sa.P, (const int32_t*)used, idx, gate,
                        reinterpret_cast<uint16_t*>(wsb + w.off_S), T, k, p->r, w.Kext, Npad, w.tile, w.n_su,
                        w.total_ks, w.ksg);
        if (rc != ADAFUSE_OK) return rc;
    }

    // Accumulators: two of H * Npad columns (Npad <= 256 / H).
    uint32_t accs = 32;
    while (accs < (uint32_t)(Npad * H)) accs <<= 1;
    const uint32_t stage_bytes = kAChunkBytes * H + (uint32_t)Npad * 128u;
    const int ST = std::min(kMaxStages, (int)((kSmemMax - 2048u) / stage_bytes));
    if (ST < 2 || 2 * accs > 512) return ADAFUSE_ERR_UNSUPPORTED;
    const uint32_t smem = (uint32_t)ST * stage_bytes + 1024u + 1024u;
    const int64_t n_sh = w.fused ? w.n_su * w.n_tt : 0;
    const int64_t n_apply = w.n_grp * w.nsplit;
    if (n_sh + n_apply > 0x7fffffff) return ADAFUSE_ERR_UNSUPPORTED;
    if (w.nsplit > 1 && H != 1) return ADAFUSE_ERR_UNSUPPORTED;     // never: splits imply the shortest units
    ApplyArgs a{};
    a.lins = p->d_desc;
    a.maps = p->d_maps;
    a.xmaps = xmaps;
    a.y_ptrs = yp;
    a.used = used;
    a.order = p->d_apply_order[w.shape];
    a.sched = p->d_sched;
    a.idx = idx;
    a.gate = gate;
    a.S = reinterpret_cast<uint16_t*>(wsb + w.off_S);
    a.P = reinterpret_cast<float*>(wsb + w.off_P);
    a.scnt = reinterpret_cast<int32_t*>(wsb + w.off_scnt);
    a.ready = reinterpret_cast<int32_t*>(wsb + w.off_ready);
    a.n_units = (int32_t)p->apply_units[w.shape];
    a.Kext = w.Kext;
    a.tile = w.tile;
    a.Mt = w.Mt;
    a.n_sh = (int32_t)n_sh;
    a.n_su = (int32_t)w.n_su;
    a.total_ks = w.total_ks;
    a.ksg = w.ksg;
    a.box_rows = p->a_box_rows;
    a.run_max = p->a_run_max;
    a.nsplit = w.nsplit;
    a.bcols = p->b_box_cols;
    a.stall = (p->flags & ADAFUSE_PLAN_TEST_STALL) ? 1 : 0;
    a.y_f32 = (p->flags & ADAFUSE_PLAN_Y_F32) ? 1 : 0;
    a.Yp = w.nsplit > 1 ? reinterpret_cast<float*>(wsb + w.off_Yp) : nullptr;
    a.cnt = w.nsplit > 1 ? reinterpret_cast<int32_t*>(wsb + w.off_cnt) : nullptr;
    a.status = p->d_status;
    a.T = T;
    a.k = k;
    a.n_lin = p->n_lin;
    a.r = p->r;
    a.n_tt = w.n_tt;
    a.Npad = Npad;
    a.stage_bytes = stage_bytes;
    a.acc_stride = accs;
    a.tmem_cols = 2 * accs;
    a.ST = ST;
    a.off_bar = (uint32_t)ST * stage_bytes;
    const int grid = (int)std::min<int64_t>(p->num_sms, n_sh + n_apply);
    p->last_launches = w.fused ? 2 : 4;
    if (w.fused) {
        if (H != 1) return ADAFUSE_ERR_UNSUPPORTED;     // never: fewer units than SMs imply the shortest units
        return launch_apply_fused<1, true>(a, smem, grid, s);
    }
    switch (H) {
    case 1: return launch_apply_fused<1, false>(a, smem, grid, s);
    case 2: return launch_apply_fused<2, false>(a, smem, grid, s);
    default: return launch_apply_fused<4, false>(a, smem, grid, s);
    }
}
}  // namespace

// y_l must be aligned to its element: 2 bytes (bf16), 4 with ADAFUSE_PLAN_Y_F32.
uintptr_t y_align_mask(const Plan* p) { return (p->flags & ADAFUSE_PLAN_Y_F32) ? 3u : 1u; }

size_t apply_workspace_bytes(const Plan* p, int64_t T, int32_t k)
{
    return ws_layout(p, T, k).total;
}

size_t apply_call_bytes(int n_lin)
{
    return (size_t)(n_lin + 1) * sizeof(CUtensorMap) + (size_t)n_lin * 2 * sizeof(void*);
}

int launch_apply(Plan* p, const void* const* x_ptrs, void* const* y_ptrs, int64_t T, const int32_t* idx,
                 const float* gate, int32_t k, void* ws, size_t ws_bytes, cudaStream_t s)
{
    const WsLayout w = ws_layout(p, T, k);
    if (ws_bytes < w.total) return ADAFUSE_ERR_WORKSPACE_TOO_SMALL;
    for (int l = 0; l < p->n_lin; ++l) {
        if (!x_ptrs[l] || !y_ptrs[l]) return ADAFUSE_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(x_ptrs[l]) & 15u) || (reinterpret_cast<uintptr_t>(y_ptrs[l]) & y_align_mask(p)))
            return ADAFUSE_ERR_UNSUPPORTED;
    }
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    uint16_t* S = reinterpret_cast<uint16_t*>(wsb + w.off_S);
    const int32_t Npad = w.Npad;

    // Per-call descriptors: rebuilt and uploaded only when something changed.
    CUtensorMap* d_maps = reinterpret_cast<CUtensorMap*>(p->d_call);
    uint8_t* d_ptrs = p->d_call + (size_t)(p->n_lin + 1) * sizeof(CUtensorMap);
    void* const* d_yp = reinterpret_cast<void* const*>(d_ptrs + sizeof(void*) * p->n_lin);
    const bool hit = p->call_valid && p->call_T == T && p->call_k == k && p->call_ws == ws &&
                     std::equal(x_ptrs, x_ptrs + p->n_lin, p->call_x.begin()) &&
                     std::equal(y_ptrs, y_ptrs + p->n_lin, p->call_y.begin());
    if (!hit) {
        std::vector<uint8_t> stage(apply_call_bytes(p->n_lin));
        CUtensorMap* hm = reinterpret_cast<CUtensorMap*>(stage.data());
        for (int l = 0; l < p->n_lin; ++l) {
            const int d_in = p->h_desc[l].d_in;
            cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
            cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
            cuuint32_t box[2] = {64, (cuuint32_t)Npad};
            if (!encode_tile_map(&hm[l], x_ptrs[l], 2, dims, strides, box)) return ADAFUSE_ERR_UNSUPPORTED;
        }
        {
            cuuint64_t dims[3] = {(cuuint64_t)(2 * w.Kext), (cuuint64_t)T, (cuuint64_t)p->n_lin};
            cuuint64_t strides[2] = {(cuuint64_t)w.Kext * 4, (cuuint64_t)T * w.Kext * 4};
            cuuint32_t box[3] = {64, (cuuint32_t)Npad, 1};
            if (!encode_tile_map(&hm[p->n_lin], S, 3, dims, strides, box)) return ADAFUSE_ERR_UNSUPPORTED;
        }
        std::memcpy(stage.data() + (size_t)(p->n_lin + 1) * sizeof(CUtensorMap), x_ptrs, sizeof(void*) * p->n_lin);
        std::memcpy(stage.data() + (size_t)(p->n_lin + 1) * sizeof(CUtensorMap) + sizeof(void*) * p->n_lin, y_ptrs,
                    sizeof(void*) * p->n_lin);
        // From pageable memory the copy is staged before the call returns, so
        // `stage` may go out of scope; it is ordered on `s` before the kernels.
        if (cudaMemcpyAsync(p->d_call, stage.data(), stage.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
            return ADAFUSE_ERR_CUDA;
        p->call_valid = true;
        p->call_T = T;
        p->call_k = k;
        p->call_ws = ws;
        p->call_x.assign(x_ptrs, x_ptrs + p->n_lin);
        p->call_y.assign(y_ptrs, y_ptrs + p->n_lin);
    }

    return launch_apply_kernels(p, w, wsb, d_maps, d_yp, idx, gate, T, k, s);
}

}  // namespace af

// ------------------------------------------------------------------ apply without allocation
//
// Scratch for adafuse_apply_noalloc: the apply workspace and the per-call TMA
// descriptor area live in this fixed device array instead of caller- or
// plan-allocated memory.  Every GPU that loads the library holds it until the
// process exits.  Host code never uses the symbol itself as an address: the
// address comes from cudaGetSymbolAddress, once per device.

namespace af {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;          // 16 MiB
constexpr int kNoAllocMaxLinears = 1024;                     // sizes the static host staging buffer below
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};
// Host staging of one call's descriptors: a static buffer (no heap), used
// under g_noalloc_stage_mu.
std::mutex g_noalloc_stage_mu;
alignas(64) uint8_t g_noalloc_stage[(kNoAllocMaxLinears + 1) * sizeof(CUtensorMap) + kNoAllocMaxLinears * sizeof(void*)];

// Device address of the scratch array on the current device, looked up the
// first time each device calls in.
int noalloc_scratch(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ADAFUSE_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return ADAFUSE_ERR_CUDA;
        g_noalloc_addr[dev] = ptr;
    }
    *out = g_noalloc_addr[dev];
    return ADAFUSE_OK;
}

}  // namespace

int launch_apply_noalloc(Plan* p, const void* const* x_ptrs, void* const* y_ptrs, int64_t T, const int32_t* idx,
                         const float* gate, int32_t k, cudaStream_t s)
{
    if (p->n_lin > kNoAllocMaxLinears) return ADAFUSE_ERR_UNSUPPORTED;
    const WsLayout w = ws_layout(p, T, k);
    const size_t desc_bytes = (((size_t)(p->n_lin + 1) * sizeof(CUtensorMap) + sizeof(void*) * p->n_lin + 255) / 256) * 256;
    if (desc_bytes + w.total > kNoAllocScratchBytes) return ADAFUSE_ERR_WORKSPACE_TOO_SMALL;
    for (int l = 0; l < p->n_lin; ++l) {
        if (!x_ptrs[l] || !y_ptrs[l]) return ADAFUSE_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(x_ptrs[l]) & 15u) || (reinterpret_cast<uintptr_t>(y_ptrs[l]) & y_align_mask(p)))
            return ADAFUSE_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc != ADAFUSE_OK) return rc;

    // Scratch layout: [descriptor area | apply workspace].
    uint8_t* d_desc = static_cast<uint8_t*>(scratch);
    CUtensorMap* d_maps = reinterpret_cast<CUtensorMap*>(d_desc);
    void* const* d_yp = reinterpret_cast<void* const*>(d_desc + (size_t)(p->n_lin + 1) * sizeof(CUtensorMap));
    uint8_t* wsb = d_desc + desc_bytes;
    uint16_t* S = reinterpret_cast<uint16_t*>(wsb + w.off_S);
    const int32_t Npad = w.Npad;

    // Descriptors for this call, staged in a static host buffer (no heap) under
    // the lock and copied from pageable memory, which the runtime stages
    // before cudaMemcpyAsync returns, so the buffer is free again at unlock.
    std::lock_guard<std::mutex> lock(g_noalloc_stage_mu);
    uint8_t* stage = g_noalloc_stage;
    CUtensorMap* hm = reinterpret_cast<CUtensorMap*>(stage);
    for (int l = 0; l < p->n_lin; ++l) {
        const int d_in = p->h_desc[l].d_in;
        cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
        cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)Npad};
        if (!encode_tile_map(&hm[l], x_ptrs[l], 2, dims, strides, box)) return ADAFUSE_ERR_UNSUPPORTED;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)(2 * w.Kext), (cuuint64_t)T, (cuuint64_t)p->n_lin};
        cuuint64_t strides[2] = {(cuuint64_t)w.Kext * 4, (cuuint64_t)T * w.Kext * 4};
        cuuint32_t box[3] = {64, (cuuint32_t)Npad, 1};
        if (!encode_tile_map(&hm[p->n_lin], S, 3, dims, strides, box)) return ADAFUSE_ERR_UNSUPPORTED;
    }
    const size_t map_bytes = (size_t)(p->n_lin + 1) * sizeof(CUtensorMap);
    std::memcpy(stage + map_bytes, y_ptrs, sizeof(void*) * p->n_lin);
    if (cudaMemcpyAsync(d_desc, stage, map_bytes + sizeof(void*) * p->n_lin, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return ADAFUSE_ERR_CUDA;

    return launch_apply_kernels(p, w, wsb, d_maps, d_yp, idx, gate, T, k, s);
}

size_t apply_noalloc_limit_bytes() { return kNoAllocScratchBytes; }

}  // namespace af

extern "C" int adafuse_apply_noalloc(adafuse_plan* plan, const void* const* x_ptrs, void* const* y_ptrs, int64_t T,
                                     const int32_t* idx, const float* gate, int32_t k, adafuse_stream_t stream)
{
    if (!plan || !x_ptrs || !y_ptrs || !idx || !gate || T < 1) return ADAFUSE_ERR_INVALID_ARG;
    if (k < 1 || k > plan->E) return ADAFUSE_ERR_UNSUPPORTED;
    if (T * (int64_t)k > 0x7fffffff) return ADAFUSE_ERR_UNSUPPORTED;
    return af::launch_apply_noalloc(plan, x_ptrs, y_ptrs, T, idx, gate, k, (cudaStream_t)stream);
}
