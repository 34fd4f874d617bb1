// Per-token activation quantisation: fp16 A [M, K] -> int8 codes [M, K] and an fp32 scale per row.
//
// "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method: the activations'
// quantisation parameters are computed from the activation matrix itself at inference time, one
// scale per token, 8-bit for W4A8 and 4-bit for W4A4. The quantiser is the symmetric one with L
// levels each side (127 or 7), evaluated in fp32 with round to nearest: inv = L / max|a|,
// q = round-half-even(a * inv) clamped to [-L, L], sa = max|a| / L; a row of zeros gives q = 0
// and sa = 0. It is the step before the layer on int8 tensor cores, whose activation operand it
// produces: 4-bit codes are held unpacked, one per int8 (tcgen05 has no 4-bit integer MMA).
//
// One CTA per row, 256 threads: 16-byte loads of 8 halves, a warp-shuffle and shared-memory
// maximum, then a second pass over the row (now in L1/L2) that writes 8 codes per thread and
// step as one 8-byte store. The work is bound by HBM: 2K bytes read and K + 4 written per row.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "wq_internal.h"

namespace wq {

constexpr int kActQuantThreads = 256;

__device__ __forceinline__ float max_abs8(uint4 v, float m) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float inv, int L) {
    auto q = [inv, L](float x) {
        int v = __float2int_rn(__fmul_rn(x, inv));
        v = v > L ? L : (v < -L ? -L : v);
        return static_cast<uint32_t>(v) & 0xFFu;
    };
    return q(a) | (q(b) << 8) | (q(c) << 16) | (q(d) << 24);
}

__global__ void __launch_bounds__(kActQuantThreads) quantize_act_kernel(const uint16_t* __restrict__ A, int K, int L,
                                                                         int8_t* __restrict__ Aq,
                                                                         float* __restrict__ sa) {
    __shared__ float warp_max[kActQuantThreads / 32];
    const int m = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(A + static_cast<size_t>(m) * K);
    const int vecs = K / 8;
    float amax = 0.0f;
    for (int i = threadIdx.x; i < vecs; i += kActQuantThreads) amax = max_abs8(__ldg(row + i), amax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < kActQuantThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
    // fp32 divisions, round to nearest (the quantiser's definition, not an approximation)
    const float levels = static_cast<float>(L);
    const float inv = amax > 0.0f ? __fdiv_rn(levels, amax) : 0.0f;
    if (threadIdx.x == 0) sa[m] = amax > 0.0f ? __fdiv_rn(amax, levels) : 0.0f;
    uint2* out = reinterpret_cast<uint2*>(Aq + static_cast<size_t>(m) * K);
    for (int i = threadIdx.x; i < vecs; i += kActQuantThreads) {
        const uint4 v = __ldg(row + i);
        const __half2* h = reinterpret_cast<const __half2*>(&v);
        const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
        const float2 f2 = __half22float2(h[2]), f3 = __half22float2(h[3]);
        out[i] = make_uint2(quant4(f0.x, f0.y, f1.x, f1.y, inv, L), quant4(f2.x, f2.y, f3.x, f3.y, inv, L));
    }
}

int launch_quantize_act(const uint16_t* A, int M, int K, int bits, int8_t* Aq, float* sa, cudaStream_t st) {
    if (M == 0) return 0;
    quantize_act_kernel<<<M, kActQuantThreads, 0, st>>>(A, K, (1 << (bits - 1)) - 1, Aq, sa);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wq
