// The layout pass: reorder 4-bit codes, group scales and (asymmetric groups) zero points into
// the blobs the GEMM streams, and its inverse (a test aid). Layout: see wq_layout.h.
#include <cuda_runtime.h>
#include <cstdint>

#include "wq_internal.h"

namespace wq {

template <bool kW4A8>
__device__ __forceinline__ int nibble_pos(int j) {
    // W4A16: code j -> position (0,4,1,5,2,6,3,7)[j];  W4A8: (0,2,4,6,1,3,5,7)[j]
    return kW4A8 ? ((j & 3) * 2 + (j >> 2)) : ((j >> 1) + 4 * (j & 1));
}

template <bool kW4A8>
__device__ __forceinline__ uint32_t permute_word(uint32_t src) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) out |= ((src >> (4 * j)) & 0xFu) << (4 * nibble_pos<kW4A8>(j));
    return out;
}

template <bool kW4A8>
__device__ __forceinline__ uint32_t unpermute_word(uint32_t src) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) out |= ((src >> (4 * nibble_pos<kW4A8>(j))) & 0xFu) << (4 * j);
    return out;
}

// One thread per (blob, h*2+v, r): four words of one column, rows 32 apart in the blob.
template <bool kW4A8>
__global__ void prepack_codes_kernel(const uint32_t* __restrict__ Q, int N, int KT, long long total,
                                     uint8_t* __restrict__ wp, size_t blob_bytes) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int hv = static_cast<int>((idx / kTileN) % 4);
    const long long blob = idx / (4 * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const long long row = static_cast<long long>(kt) * 16 + hv * 4 + i;  // row of Q (8 codes each)
        w[i] = (n < N) ? permute_word<kW4A8>(__ldg(Q + row * N + n)) : 0x88888888u;
    }
    uint4* dst = reinterpret_cast<uint4*>(wp + blob * blob_bytes + (static_cast<size_t>(hv) * kTileN + r) * 16);
    *dst = make_uint4(w[0], w[1], w[2], w[3]);
}

template <bool kW4A8>
__global__ void unpack_codes_kernel(const uint8_t* __restrict__ wp, int N, int KT, long long total,
                                    uint32_t* __restrict__ Q, size_t blob_bytes) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int hv = static_cast<int>((idx / kTileN) % 4);
    const long long blob = idx / (4 * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    if (n >= N) return;
    const uint4 v = *reinterpret_cast<const uint4*>(wp + blob * blob_bytes + (static_cast<size_t>(hv) * kTileN + r) * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const long long row = static_cast<long long>(kt) * 16 + hv * 4 + i;
        Q[row * N + n] = unpermute_word<kW4A8>(w[i]);
    }
}

// One thread per (blob, slot, r): copy one scale into the blob's scale rows.
__global__ void prepack_scales_kernel(const uint16_t* __restrict__ s, int N, int KT, int g, int slots,
                                      long long total, uint8_t* __restrict__ wp, size_t blob_bytes) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const long long grp = (static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g) / g;
    const uint16_t v = (n < N) ? s[grp * N + n] : static_cast<uint16_t>(0);
    reinterpret_cast<uint16_t*>(wp + blob * blob_bytes + kCodeBytes)[u * kTileN + r] = v;
}

__global__ void unpack_scales_kernel(const uint8_t* __restrict__ wp, int N, int KT, int g, int slots,
                                     long long total, uint16_t* __restrict__ s, size_t blob_bytes) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const long long row0 = static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g;
    if (n >= N || row0 % g != 0) return;  // a group larger than a blob is written by its first blob only
    s[(row0 / g) * N + n] = reinterpret_cast<const uint16_t*>(wp + blob * blob_bytes + kCodeBytes)[u * kTileN + r];
}

// One thread per (blob, slot, r): copy one zero point into the blob's zero rows (asymmetric groups).
__global__ void prepack_zeros_kernel(const uint8_t* __restrict__ z, int N, int KT, int g, int slots, long long total,
                                     uint8_t* __restrict__ wp, size_t blob_bytes, size_t zoff) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const long long grp = (static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g) / g;
    wp[blob * blob_bytes + zoff + u * kTileN + r] = (n < N) ? z[grp * N + n] : static_cast<uint8_t>(8);
}

__global__ void unpack_zeros_kernel(const uint8_t* __restrict__ wp, int N, int KT, int g, int slots, long long total,
                                    uint8_t* __restrict__ z, size_t blob_bytes, size_t zoff) {
    long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const long long row0 = static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g;
    if (n >= N || row0 % g != 0) return;  // a group larger than a blob is written by its first blob only
    z[(row0 / g) * N + n] = wp[blob * blob_bytes + zoff + u * kTileN + r];
}

__global__ void channel_tail_kernel(const uint16_t* __restrict__ s, int N, int padded, int tail_elems,
                                    uint16_t* __restrict__ tail) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < tail_elems) tail[i] = (i < N) ? s[i] : static_cast<uint16_t>(0);
    (void)padded;
}

__global__ void channel_untail_kernel(const uint16_t* __restrict__ tail, int N, uint16_t* __restrict__ s) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < N) s[i] = tail[i];
}

static inline unsigned blocks_for(long long total, int threads) {
    return static_cast<unsigned>((total + threads - 1) / threads);
}

int launch_prepack(const int32_t* Q, const uint16_t* s, const uint8_t* z, int K, int N, int g, void* Wp,
                   cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    const size_t blob = slots > 0 ? (z ? blob_bytes_w4a16_zp(slots) : blob_bytes_w4a16(slots))
                                  : static_cast<size_t>(kCodeBytes);
    uint8_t* wp = static_cast<uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 4 * kTileN;
    prepack_codes_kernel<false><<<blocks_for(tc, 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(Q), N, KT, tc,
                                                                      wp, blob);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        prepack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(s, N, KT, g, slots, ts, wp, blob);
        if (z)
            prepack_zeros_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(z, N, KT, g, slots, ts, wp, blob,
                                                                       blob_bytes_w4a16(slots));
    } else {
        const int tail_elems = static_cast<int>(channel_tail_bytes(N) / 2);
        channel_tail_kernel<<<blocks_for(tail_elems, 256), 256, 0, st>>>(
            s, N, NT * kTileN, tail_elems, reinterpret_cast<uint16_t*>(wp + nblob * blob));
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_prepack_w4a8(const int32_t* Q, int K, int N, void* Wp, cudaStream_t st) {
    const int KT = K / kTileK, NT = n_tiles(N);
    const long long tc = static_cast<long long>(NT) * KT * 4 * kTileN;
    prepack_codes_kernel<true><<<blocks_for(tc, 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(Q), N, KT, tc,
                                                                     static_cast<uint8_t*>(Wp), kCodeBytes);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_unpack(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, uint8_t* z, cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    const size_t blob = slots > 0 ? (z ? blob_bytes_w4a16_zp(slots) : blob_bytes_w4a16(slots))
                                  : static_cast<size_t>(kCodeBytes);
    const uint8_t* wp = static_cast<const uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 4 * kTileN;
    unpack_codes_kernel<false><<<blocks_for(tc, 256), 256, 0, st>>>(wp, N, KT, tc, reinterpret_cast<uint32_t*>(Q),
                                                                     blob);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        unpack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(wp, N, KT, g, slots, ts, s, blob);
        if (z)
            unpack_zeros_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(wp, N, KT, g, slots, ts, z, blob,
                                                                      blob_bytes_w4a16(slots));
    } else {
        channel_untail_kernel<<<blocks_for(N, 256), 256, 0, st>>>(
            reinterpret_cast<const uint16_t*>(wp + nblob * blob), N, s);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_unpack_w4a8(const void* Wp, int K, int N, int32_t* Q, cudaStream_t st) {
    const int KT = K / kTileK, NT = n_tiles(N);
    const long long tc = static_cast<long long>(NT) * KT * 4 * kTileN;
    unpack_codes_kernel<true><<<blocks_for(tc, 256), 256, 0, st>>>(static_cast<const uint8_t*>(Wp), N, KT, tc,
                                                                    reinterpret_cast<uint32_t*>(Q), kCodeBytes);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wq
