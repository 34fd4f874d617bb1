// Act order: groups whose rows are scattered along K (row k in group g_idx[k]).
//
// "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method: fine-grained
// groups with one scale (and zero point) each. When the rows of a group are not consecutive
// (GPTQ-style act-order checkpoints), taking the weight's rows and the activations' columns in
// an order perm with g_idx[perm[i]] = i / g makes every group a run of g rows again and leaves
// y = A . W unchanged: sum_k a_k w_k = sum_i a_perm[i] w_perm[i]. So the weight is reordered
// once, by the layout pass, and each call gathers the activations' columns in the same order
// before the grouped layer runs.
//
// permute_codes_kernel: one thread per output word (8 rows of one column) of the reordered
// codes; the threads of a warp take adjacent columns, so every read of Q is coalesced.
// permute_act_kernel: one thread per 8 consecutive output columns of one row: two 16-byte
// loads of perm, eight 2-byte gathers from the row (which stays in L1/L2 while its CTAs run),
// one 16-byte store. An index outside [0, K) is never dereferenced: the element becomes 0 and
// the device status word records WQ_ERR_INVALID_ARG. HBM-bound: 2MK bytes read, 2MK written.
#include <cuda_runtime.h>
#include <cstdint>

#include "wq_internal.h"

namespace wq {

constexpr int kPermThreads = 256;

__global__ void permute_codes_kernel(const uint32_t* __restrict__ Q, const int32_t* __restrict__ perm, int K, int N,
                                     uint32_t* __restrict__ Qp) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    const long long words = static_cast<long long>(K / 8) * N;
    if (idx >= words) return;
    const int n = static_cast<int>(idx % N);
    const int i8 = static_cast<int>(idx / N);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = perm[8 * i8 + j];  // validated on the host: 0 <= r < K
        const uint32_t code = (Q[static_cast<size_t>(r >> 3) * N + n] >> (4 * (r & 7))) & 0xFu;
        w |= code << (4 * j);
    }
    Qp[idx] = w;
}

__global__ void __launch_bounds__(kPermThreads) permute_act_kernel(const uint16_t* __restrict__ A,
                                                                   const int32_t* __restrict__ perm, int K,
                                                                   int blocks_per_row, uint16_t* __restrict__ Ap,
                                                                   int* __restrict__ status) {
    const long long m = blockIdx.x / blocks_per_row;
    const int i0 = ((blockIdx.x % blocks_per_row) * kPermThreads + threadIdx.x) * 8;
    if (i0 >= K) return;
    const int4 p0 = *reinterpret_cast<const int4*>(perm + i0);
    const int4 p1 = *reinterpret_cast<const int4*>(perm + i0 + 4);
    const int p[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const uint16_t* row = A + m * K;
    uint16_t v[8];
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const bool ok = static_cast<unsigned>(p[j]) < static_cast<unsigned>(K);
        v[j] = ok ? __ldg(row + p[j]) : static_cast<uint16_t>(0);
        bad |= !ok;
    }
    if (bad) atomicCAS(status, 0, 1 /* WQ_ERR_INVALID_ARG */);
    uint4 out;
    out.x = v[0] | (static_cast<uint32_t>(v[1]) << 16);
    out.y = v[2] | (static_cast<uint32_t>(v[3]) << 16);
    out.z = v[4] | (static_cast<uint32_t>(v[5]) << 16);
    out.w = v[6] | (static_cast<uint32_t>(v[7]) << 16);
    *reinterpret_cast<uint4*>(Ap + m * K + i0) = out;
}

int launch_permute_codes(const int32_t* Q, const int32_t* perm, int K, int N, int32_t* Qp, cudaStream_t st) {
    const long long words = static_cast<long long>(K / 8) * N;
    const unsigned blocks = static_cast<unsigned>((words + kPermThreads - 1) / kPermThreads);
    permute_codes_kernel<<<blocks, kPermThreads, 0, st>>>(reinterpret_cast<const uint32_t*>(Q), perm, K, N,
                                                          reinterpret_cast<uint32_t*>(Qp));
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_permute_act(const uint16_t* A, const int32_t* perm, int M, int K, uint16_t* Ap, int* status,
                       cudaStream_t st) {
    if (M == 0) return 0;
    const int per_row = (K / 8 + kPermThreads - 1) / kPermThreads;
    const long long blocks = static_cast<long long>(M) * per_row;
    permute_act_kernel<<<static_cast<unsigned>(blocks), kPermThreads, 0, st>>>(A, perm, K, per_row, Ap, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wq
