/*
 * adafuse.h -- C ABI of libadafuse.so, a B200 (sm_100a) implementation of the
 * data-parallel hot path of AdaFuse ("AdaFuse: Accelerating Dynamic Adapter
 * Inference via Token-Level Pre-Gating and Fused Kernel Optimization"):
 *
 *   pregate : token-level pre-gating -- one router at the first adapted layer
 *             picks the top-k LoRA experts of each token once, and that choice
 *             is reused by every layer (page pt section 2.A "Arquitetura de
 *             Pre-Gating por Token"; page ja section 2.1).
 *   merge   : the SGMM fused merge -- the selected adapters' down (A) and up (B)
 *             projections are concatenated and fused into the backbone weights
 *             of every targeted linear of every layer in one kernel launch,
 *             W' = W + sum_s g_s B_{e_s} A_{e_s} (page pt section 2.B "Fusao de
 *             Adaptadores e Kernel SGMM"; page ja section 2.2 steps 1-3).
 *   switch  : undo the previous token's fusion and fuse the current one in one
 *             pass (page pt section 2.B, "Troca Eficiente").
 *   apply   : the segmented-gather ("Segmented Gather Matrix Multiplication",
 *             page pt section 2.B) unmerged form for batches whose sequences
 *             picked different adapters, y = x W^T + sum_s g_s (x A_s^T) B_s^T.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *     parameter says "host".  bf16 is IEEE bfloat16 (uint16 storage).
 *   - W of a linear is [d_out, d_in] row-major (an nn.Linear weight); adapter
 *     e has A_e [r, d_in] and B_e [d_out, r], both row-major; the LoRA scale is
 *     1 (fold any alpha/r into B).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and allocates nothing; only adafuse_plan_create
 *     allocates (its device tables), and adafuse_plan_destroy frees them.
 *   - Return value: ADAFUSE_OK or one of the error codes below.  Argument
 *     errors are detected on the host before anything is launched.  No C++
 *     exception crosses this boundary.  Errors found on the device (an expert
 *     index outside [0, E), a wait that timed out) never trap: the kernel
 *     skips the offending slot or gives up the wait, sets a bit in the plan's
 *     status word and finishes; read it with adafuse_plan_status.
 *   - A plan may be used from one stream at a time.
 *   - The library's kernels are launched with programmatic stream
 *     serialization (programmatic dependent launch): each one may start while
 *     the previous kernel on the stream is still running. Before any
 *     global-memory access it waits until that kernel has completed, so work
 *     queued ahead of a call is ordered as usual. Each library kernel lets
 *     the next kernel of the stream launch early. A caller's kernel launched
 *     normally after a call waits for the call to finish, as always. A
 *     caller's kernel launched with the programmatic-serialization
 *     attribute must execute griddepcontrol.wait (cudaGridDependencySynchronize)
 *     before it reads the call's outputs.
 */
#ifndef ADAFUSE_H
#define ADAFUSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ADAFUSE_API __attribute__((visibility("default")))
#else
#define ADAFUSE_API
#endif

typedef struct CUstream_st* adafuse_stream_t;   /* same type as cudaStream_t */

/* ---- return codes ---- */
#define ADAFUSE_OK                      0
#define ADAFUSE_ERR_INVALID_ARG         1   /* null pointer, negative size, ... */
#define ADAFUSE_ERR_UNSUPPORTED         2   /* outside the supported envelope (see each call) */
#define ADAFUSE_ERR_WORKSPACE_TOO_SMALL 3
#define ADAFUSE_ERR_CUDA                4   /* a CUDA runtime/driver call failed */
#define ADAFUSE_ERR_TIMEOUT             5   /* a device-side wait gave up (status word) */
#define ADAFUSE_ERR_DEVICE              6   /* no usable sm_100 device */

/* ---- flags ---- */
#define ADAFUSE_RENORM     (1u << 0)   /* pregate: divide the k gates by their sum */
#define ADAFUSE_POOL_MEAN  (1u << 1)   /* pregate: one decision for the mean of the T rows */

/* ---- plan flags ---- */
/* The apply of this plan writes every y_l as fp32 [T, d_out] (4-byte aligned),
 * the unrounded fp32 accumulator of x W^T + the LoRA term, instead of bf16.
 * For the row-parallel shards of tensor parallelism (attention output and
 * down projections split along d_in): each rank's y is a partial sum, and
 * rounding it to bf16 before the ranks' partials are added loses up to half a
 * bf16 ulp per partial, more than the output tolerance where the partials
 * cancel.  With this flag the partials are added in fp32 (the all-reduce) and
 * rounded once, by adafuse_round_bf16.  Merge and switch are unaffected. */
#define ADAFUSE_PLAN_Y_F32       (1u << 0)
/* Test hook for the failure path: every fused merge, switch or apply on a
 * plan created with this flag withholds the first shared-memory stage of CTA 0
 * of the merge or of the fused apply kernel, so that CTA's pipeline wait runs
 * out (after about 1.5 s) instead of the data arriving.  The launch then
 * completes with ADAFUSE_STATUS_TIMEOUT set and W_out (or y) incomplete, while
 * the GPU context stays usable.  Never set it outside tests. */
#define ADAFUSE_PLAN_TEST_STALL  (1u << 31)

/* ---- device status bits (adafuse_plan_status) ---- */
#define ADAFUSE_STATUS_BAD_INDEX  (1 << 0)   /* an expert index was outside [0, E); slot skipped */
#define ADAFUSE_STATUS_TIMEOUT    (1 << 1)   /* a pipeline wait exceeded its limit; output invalid */

/* ---- limits ---- */
#define ADAFUSE_MAX_E      32    /* experts per router (one warp lane each) */
#define ADAFUSE_MAX_SLOTS  64    /* selection slots in one merge pass: k (merge), 2k (switch) */
#define ADAFUSE_MAX_KR     256   /* k*r (merge), 2*k*r (switch) */

/* One targeted linear of the backbone. */
typedef struct {
    const void* W;              /* bf16 [d_out, d_in] row-major, 16-byte aligned */
    void*       W_out;          /* bf16 [d_out, d_in] row-major, 16-byte aligned; may equal W */
    const void* A;              /* bf16; A_e = A + e*a_expert_stride, [r, d_in] row-major */
    const void* B;              /* bf16; B_e = B + e*b_expert_stride, [d_out, r] row-major */
    int32_t     d_out, d_in;    /* both multiples of 8, >= 8 */
    int64_t     a_expert_stride;    /* elements, multiple of 8, >= r*d_in */
    int64_t     b_expert_stride;    /* elements, multiple of 8, >= d_out*r */
} adafuse_linear;

typedef struct adafuse_plan adafuse_plan;     /* opaque, library-owned */

/*
 * Build a plan for n_lin linears sharing E adapters of rank r: the device
 * table of linears, the TMA descriptors of W, W_out and B, the per-CTA work
 * split of merge and apply, and the status word.  Everything is built once
 * here so that the hot calls do no host work beyond a launch.
 * The `lins` array (host) is copied; the tensors it points to must outlive the
 * plan.  Uses the current CUDA device.  `flags`: 0, or ADAFUSE_PLAN_Y_F32
 * and / or ADAFUSE_PLAN_TEST_STALL.
 * Errors: INVALID_ARG (null pointers, n_lin < 1, other flags), UNSUPPORTED (E outside
 * [1, 32], r not a multiple of 8 or r > 256, d_out/d_in not multiples of 8,
 * misaligned pointers or strides), DEVICE (no sm_100 GPU), CUDA.
 */
ADAFUSE_API int adafuse_plan_create(adafuse_plan** out, const adafuse_linear* lins, int32_t n_lin,
                        int32_t E, int32_t r, uint32_t flags);

/* Free a plan's device tables (synchronises the device).  NULL is a no-op. */
ADAFUSE_API void adafuse_plan_destroy(adafuse_plan* plan);

/*
 * Token-level pre-gating (page pt section 2.A; page ja section 2.1): for each
 * of the T rows of x, logits z_e = sum_j x_j W_r[e, j] (+ b_r[e]) over all E
 * experts, then the k experts with the largest logits (equal logits: lower
 * index first; NaN ranks last) in that order, and their softmax
 * probabilities over all E experts as gates.
 *   x            bf16 [T, H], consecutive rows x_row_stride elements apart (>= H);
 *                no alignment beyond 2 bytes is required
 *   W_r          fp32 [E, H] row-major;  b_r  fp32 [E] or NULL
 *   idx          int32 [T, k] out (ADAFUSE_POOL_MEAN: [1, k])
 *   gate         fp32  [T, k] out (ADAFUSE_POOL_MEAN: [1, k])
 *   flags        ADAFUSE_RENORM: gates divided by their sum;
 *                ADAFUSE_POOL_MEAN: route the mean of the T rows once (a
 *                sequence-level decision).
 * The logits are computed in fp32 exactly as written above: each product
 * rounded to fp32, added in ascending j, bias last; so the selection is a
 * deterministic function of the inputs.  Cost is the launch plus H serial adds.
 * Errors: INVALID_ARG (null, T < 1, H < 1, stride < H), UNSUPPORTED (E > 32,
 * k < 1 or k > E).
 */
ADAFUSE_API int adafuse_pregate(const void* x, int64_t T, int32_t H, int64_t x_row_stride,
                    const float* W_r, const float* b_r, int32_t E, int32_t k,
                    uint32_t flags, int32_t* idx, float* gate, adafuse_stream_t stream);

/*
 * Fused all-layer merge (page pt section 2.B; page ja section 2.2): for every
 * linear of the plan, W_out = bf16_rne(W + sum_{s<k} gate[s] B_{idx[s]} A_{idx[s]}),
 * accumulated in fp32, in ONE kernel launch over all linears.  The gates are
 * folded into one factor of the concatenated product, rounded to bf16: into
 * the B rows (g_s B_{e_s}) when k*r <= 128, into the A rows (g_s A_{e_s})
 * when k*r is above 128 (up to 256).  The rank-(k*r) contraction runs on the
 * tensor cores, W streams through shared memory by TMA.  idx int32 [k], gate fp32 [k] (device; e.g. row 0 of pregate's output).
 * In place when W_out == W.
 * Errors: INVALID_ARG, UNSUPPORTED (k < 1, k > E, k*r > 256).
 */
ADAFUSE_API int adafuse_merge(adafuse_plan* plan, const int32_t* idx, const float* gate, int32_t k,
                  adafuse_stream_t stream);

/*
 * Adapter switch in place (page pt section 2.B, "Troca Eficiente": undo the
 * previous fusion and fuse the current one in parallel): for every linear,
 * W_out = bf16_rne(W_out + sum_s g_new[s] B A - sum_s g_old[s] B A), one pass,
 * rank 2*k*r.  W is not read.  When the two selections are identical (same
 * indices and gate bits, in order) the kernel returns at once and W_out is
 * left untouched.  bf16 rounding makes switch(old -> new) differ from a fresh
 * merge(new) by at most one bf16 rounding step per element.
 * Errors: as adafuse_merge, with 2*k*r <= 256.
 */
ADAFUSE_API int adafuse_switch(adafuse_plan* plan, const int32_t* idx_new, const float* gate_new,
                   const int32_t* idx_old, const float* gate_old, int32_t k,
                   adafuse_stream_t stream);

/*
 * Baseline for the merge (the ablation "simple fusion without SGMM", page pt
 * section 4, Estudo de Ablacao; page ja section 4): the same result as
 * adafuse_merge, computed with one kernel launch per linear, CUDA-core FMAs
 * and no shared-memory pipeline.  For comparison only.
 */
ADAFUSE_API int adafuse_merge_per_linear(adafuse_plan* plan, const int32_t* idx, const float* gate,
                             int32_t k, adafuse_stream_t stream);

/*
 * Segments of a mixed batch ("Segmented Gather"): the T*k (token, slot) pairs,
 * numbered p = t*k + s, stably sorted by expert.  Outputs (device):
 *   offsets int32 [E+1]   expert e's pairs are perm[offsets[e] .. offsets[e+1])
 *   perm    int32 [T*k]   pair ids; entries past offsets[E] are unspecified
 *   used    int32 [E+1]   used[0] = U, the number of experts with a non-empty
 *                         segment; used[1..U] those experts in ascending order
 *   status  int32 [1]     (nullable) ADAFUSE_STATUS_BAD_INDEX is OR-ed in when an
 *                         index is outside [0, E); such pairs are left out
 * One launch of one CTA.  Errors: INVALID_ARG, UNSUPPORTED (E > 32).
 */
ADAFUSE_API int adafuse_segments(const int32_t* idx, int64_t T, int32_t k, int32_t E,
                     int32_t* offsets, int32_t* perm, int32_t* used, int32_t* status,
                     adafuse_stream_t stream);

/* Bytes of device workspace adafuse_apply needs for T tokens and top-k. */
ADAFUSE_API size_t adafuse_apply_workspace_bytes(const adafuse_plan* plan, int64_t T, int32_t k);

/*
 * Segmented-gather apply, unmerged, for every linear of the plan:
 *   y_l[t, :] = bf16_rne( x_l[t, :] W_l^T + sum_s gate[t,s] (x_l[t, :] A_{idx[t,s]}^T) B_{idx[t,s]}^T )
 * with fp32 accumulation.  Two launches, whatever the number of linears: the
 * segment build (stable sort of the pairs by expert; gives the U experts the
 * batch uses), then one persistent tensor-core kernel over all linears that
 * runs the shrink first (the used experts' A rows times x^T, split over
 * 1024-column K-slices, 256 for small plans; the last slice of each tile to
 * finish adds the slices in order, applies the gates and keeps the result as
 * a pair of bf16 values whose sum is the fp32 result), then streams W once
 * and adds the expand (the used experts' B rows against both halves of the
 * shrink) into the same fp32 accumulator, each linear's expand starting once
 * its shrink is complete.
 *   x_ptrs   HOST array [n_lin] of device pointers, x_l bf16 [T, d_in_l] row-major,
 *            16-byte aligned
 *   y_ptrs   HOST array [n_lin] of device pointers, y_l bf16 [T, d_out_l] row-major
 *            (fp32, 4-byte aligned, for a plan created with ADAFUSE_PLAN_Y_F32)
 *   idx/gate int32 / fp32 [T, k] (device), e.g. pregate's output
 *   workspace device, >= adafuse_apply_workspace_bytes(plan, T, k), 256-byte aligned
 * The call builds TMA descriptors for the x_l and the workspace and uploads
 * them (with the pointer tables) on `stream`; they are kept in the plan and
 * rebuilt only when the pointers, T, k or the workspace differ from the
 * previous call, so a serving loop that reuses its buffers does no host work
 * beyond the two launches.  The apply kernel's work units cover 512, 256 or 128 output
 * rows with token tiles of 64, 128 or 256 (taller units for smaller T, as long
 * as the plan has two units per SM; with fewer than one per SM, units are
 * split along K and their fp32 partials added in a fixed order); T larger
 * than 256 streams W once per tile.  Each row of idx should hold distinct
 * experts (as pregate's does); a repeated expert adds its gates.
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL, UNSUPPORTED (k < 1, k > E,
 * misaligned x_l).
 */
ADAFUSE_API int adafuse_apply(adafuse_plan* plan, const void* const* x_ptrs, void* const* y_ptrs,
                  int64_t T, const int32_t* idx, const float* gate, int32_t k,
                  void* workspace, size_t ws_bytes, adafuse_stream_t stream);

/*
 * adafuse_apply without any allocation.  (No counterpart in the paper: this is
 * a convenience of this library.)
 *
 * Computes exactly what adafuse_apply computes, through the same kernels, but
 * takes no workspace: the workspace and the per-call TMA descriptors live in a
 * fixed 16 MiB array inside the library's own device memory.  It is for
 * callers that cannot allocate device memory on their hot path -- a runtime
 * that hands all GPU memory to its own pool at start-up and has none left to
 * give out, or code that must not call cudaMalloc there because cudaMalloc can
 * synchronise the device -- and for callers that would rather not manage a
 * workspace at all.  It calls no cudaMalloc, cudaFree or other allocating
 * routine, on the device or the host.
 *   - Limit: the call needs adafuse_apply_workspace_bytes(plan, T, k) plus
 *     (n_lin + 1) * 128 + n_lin * 8 bytes of descriptors, rounded up to a
 *     multiple of 256; if that exceeds 16 MiB it
 *     returns ADAFUSE_ERR_WORKSPACE_TOO_SMALL and launches nothing (e.g. the
 *     224-linear Llama-2-7B plan with E = 8, r = 16, top-2 fits up to T = 16).
 *     At most 1024 linears (ADAFUSE_ERR_UNSUPPORTED beyond).
 *   - The array exists on every GPU that loads the library, until the process
 *     exits, whether or not this entry point is used.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins.
 *   - Every call on a device uses the same array and leaves its contents
 *     behind; nothing in it has to start at zero, because each call writes
 *     every byte it later reads.  Calls whose work overlaps on the GPU (other
 *     streams, other plans, other threads) race on the array: the caller must
 *     order them, e.g. by issuing them on one stream.
 *   - The descriptors are rebuilt on every call (adafuse_apply caches them).
 * Arguments, outputs and other errors as adafuse_apply.
 */
ADAFUSE_API int adafuse_apply_noalloc(adafuse_plan* plan, const void* const* x_ptrs, void* const* y_ptrs,
                                      int64_t T, const int32_t* idx, const float* gate, int32_t k,
                                      adafuse_stream_t stream);

/*
 * Round fp32 values to bf16, round-to-nearest-even: out[i] = bf16_rne(in[i])
 * for i < n (values above the bf16 range become +-inf, NaN stays NaN).  The
 * last step of a tensor-parallel row-parallel apply: the ranks' fp32 partial
 * outputs (ADAFUSE_PLAN_Y_F32) are summed by the caller's all-reduce, and this
 * rounds the sum once, as the unsharded apply rounds its accumulator (page ja
 * section 2.2 computes the fused product across layers; the sharding is this
 * library's extension for multi-GPU serving).
 *   in   device fp32 [n], 4-byte aligned
 *   out  device bf16 [n], 2-byte aligned, not overlapping in
 * One launch.  Errors: INVALID_ARG (null pointer with n > 0, n < 0, misaligned or
 * overlapping buffers).  n == 0 launches nothing.
 */
ADAFUSE_API int adafuse_round_bf16(const float* in, void* out, int64_t n, adafuse_stream_t stream);

/*
 * Synchronise `stream`, read the plan's device status word into
 * *device_status (host) and clear it.  Returns ADAFUSE_ERR_TIMEOUT if the
 * TIMEOUT bit was set, else ADAFUSE_OK (a BAD_INDEX bit alone is reported in
 * *device_status only).
 */
ADAFUSE_API int adafuse_plan_status(adafuse_plan* plan, adafuse_stream_t stream, int32_t* device_status);

/* Number of kernel launches the last call on this plan made (host counter). */
ADAFUSE_API int32_t adafuse_plan_last_launches(const adafuse_plan* plan);

/* Static description of an error code. */
ADAFUSE_API const char* adafuse_strerror(int code);

/* Library version, major*10000 + minor*100 + patch. */
ADAFUSE_API int32_t adafuse_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ADAFUSE_H */
