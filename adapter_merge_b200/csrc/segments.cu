// Segment build for the mixed-batch apply ("Segmented Gather"): the T*k
// (token, slot) pairs, numbered p = t*k + s, stably sorted by expert index.
//
// One CTA.  Each thread owns a contiguous run of pairs and counts its experts;
// an exclusive scan over (expert, thread) gives every thread its write cursor
// per expert, and a second pass over the same run scatters the pair ids, so
// the order inside a segment is ascending p.  Indices outside [0, E) are left
// out and flagged.
#include "internal.h"
#include "ptx.cuh"

namespace af {

namespace {

constexpr int kSegThreads = 256;

// zero[0 .. n_zero) is cleared as well: the counters the apply kernel of the
// same call starts from (nothing else on the stream touches them in between).
__global__ void __launch_bounds__(kSegThreads) segments_kernel(const int32_t* idx, int64_t P, int32_t E,
                                                               int32_t* offsets, int32_t* perm, int32_t* used,
                                                               int32_t* status, int32_t* zero, int64_t n_zero)
{
    __shared__ int cnt[kSegThreads][kMaxE + 1];
    __shared__ int s_off[kMaxE + 1];
    const int tid = threadIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    for (int64_t i = tid; i < n_zero; i += kSegThreads) zero[i] = 0;
    const int64_t chunk = (P + kSegThreads - 1) / kSegThreads;
    const int64_t p0 = (int64_t)tid * chunk < P ? (int64_t)tid * chunk : P;
    const int64_t p1 = p0 + chunk < P ? p0 + chunk : P;
    for (int e = 0; e < E; ++e) cnt[tid][e] = 0;
    int bad = 0;
    for (int64_t p = p0; p < p1; ++p) {
        const int e = idx[p];
        if (e < 0 || e >= E) { bad = 1; continue; }
        cnt[tid][e] += 1;
    }
    __syncthreads();
    if (tid < E) {
        int run = 0;
        for (int t2 = 0; t2 < kSegThreads; ++t2) {
            const int c = cnt[t2][tid];
            cnt[t2][tid] = run;
            run += c;
        }
        s_off[tid + 1] = run;        // segment size for now
    }
    __syncthreads();
    if (tid == 0) {
        s_off[0] = 0;
        int U = 0;
        for (int e = 0; e < E; ++e) {
            const int sz = s_off[e + 1];
            s_off[e + 1] = s_off[e] + sz;
            if (sz > 0) used[1 + U++] = e;
        }
        used[0] = U;
        for (int e = 0; e <= E; ++e) offsets[e] = s_off[e];
    }
    __syncthreads();
    for (int64_t p = p0; p < p1; ++p) {
        const int e = idx[p];
        if (e < 0 || e >= E) continue;
        perm[s_off[e] + cnt[tid][e]] = (int32_t)p;
        cnt[tid][e] += 1;
    }
    if (bad && status) atomicOr(status, ADAFUSE_STATUS_BAD_INDEX);
}

}  // namespace

int launch_segments(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offsets, int32_t* perm,
                    int32_t* used, int32_t* status, cudaStream_t s, int32_t* zero, int64_t n_zero)
{
    return launch_pdl(segments_kernel, dim3(1), dim3(kSegThreads), 0, s, idx, T * k, E, offsets, perm, used,
                      status, zero, n_zero);
}

}  // namespace af

extern "C" int adafuse_segments(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                                int32_t* perm, int32_t* used, int32_t* status, adafuse_stream_t stream)
{
    if (!idx || !offsets || !perm || !used || T < 1 || k < 1) return ADAFUSE_ERR_INVALID_ARG;
    if (E < 1 || E > af::kMaxE) return ADAFUSE_ERR_UNSUPPORTED;
    if (T * (int64_t)k > 0x7fffffff) return ADAFUSE_ERR_UNSUPPORTED;
    return af::launch_segments(idx, T, k, E, offsets, perm, used, status, (cudaStream_t)stream);
}
