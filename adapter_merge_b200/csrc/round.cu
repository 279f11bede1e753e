// fp32 -> bf16 rounding (round to nearest, ties to even) of a device buffer:
// the one rounding of a tensor-parallel row-parallel apply, after the ranks'
// fp32 partial outputs have been summed by the all-reduce.
//
// HBM-bound (6 bytes moved per element): each thread converts four elements
// per step with a 16-byte load and an 8-byte store where both buffers allow
// it, over a grid of a few CTAs per SM; the ragged head and tail go one
// element at a time.
#include <cuda_bf16.h>

#include "internal.h"

namespace af {
namespace {

constexpr int kRoundThreads = 256;

__global__ void __launch_bounds__(kRoundThreads) round_bf16_kernel(const float* in, uint16_t* out, int64_t n,
                                                                   int64_t head, int64_t n_vec)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // head elements one by one, until both pointers are vector-aligned
    for (int64_t i = tid; i < head; i += stride)
        out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
    const float4* in4 = reinterpret_cast<const float4*>(in + head);
    uint2* out4 = reinterpret_cast<uint2*>(out + head);
    for (int64_t i = tid; i < n_vec; i += stride) {
        const float4 v = __ldcs(in4 + i);
        uint2 o;
        o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y)) << 16);
        o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w)) << 16);
        __stcs(out4 + i, o);
    }
    for (int64_t i = head + 4 * n_vec + tid; i < n; i += stride)
        out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
}

}  // namespace
}  // namespace af

using namespace af;

extern "C" int adafuse_round_bf16(const float* in, void* out, int64_t n, adafuse_stream_t stream)
{
    if (n < 0) return ADAFUSE_ERR_INVALID_ARG;
    if (n == 0) return ADAFUSE_OK;
    if (!in || !out) return ADAFUSE_ERR_INVALID_ARG;
    const uintptr_t pi = reinterpret_cast<uintptr_t>(in), po = reinterpret_cast<uintptr_t>(out);
    if ((pi & 3u) || (po & 1u)) return ADAFUSE_ERR_INVALID_ARG;
    if (pi < po + (uintptr_t)n * 2 && po < pi + (uintptr_t)n * 4) return ADAFUSE_ERR_INVALID_ARG;
    // The vector body needs in 16-byte and out 8-byte aligned at the same
    // element: possible only if both offsets agree modulo four elements.
    int64_t head = 0, n_vec = 0;
    const int64_t hi = (int64_t)((16 - (pi & 15u)) & 15u) / 4;     // elements until in is 16-byte aligned
    if (((po + (uintptr_t)hi * 2) & 7u) == 0 && hi <= n) {
        head = hi;
        n_vec = (n - head) / 4;
    } else {
        head = n;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t work = std::max<int64_t>(n_vec, head + (n - head - 4 * n_vec));
    const int64_t blocks = std::min<int64_t>((int64_t)sms * 8, (work + kRoundThreads - 1) / kRoundThreads);
    round_bf16_kernel<<<(unsigned)std::max<int64_t>(1, blocks), kRoundThreads, 0, (cudaStream_t)stream>>>(
        in, static_cast<uint16_t*>(out), n, head, n_vec);
    return cuda_err(cudaGetLastError());
}
