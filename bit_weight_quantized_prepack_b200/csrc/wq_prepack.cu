// The layout pass: reorder 4-bit codes, group scales and (asymmetric groups) zero points into
// the blobs the GEMM streams, and its inverse (a test aid); the same for 2:4 sparse weights
// (kept codes and their positions). Layouts: see wq_layout.h.
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
                                      long long total, uint8_t* __restrict__ wp, size_t blob_bytes, int head) {
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
    reinterpret_cast<uint16_t*>(wp + blob * blob_bytes + head)[u * kTileN + r] = v;
}

__global__ void unpack_scales_kernel(const uint8_t* __restrict__ wp, int N, int KT, int g, int slots,
                                     long long total, uint16_t* __restrict__ s, size_t blob_bytes, int head) {
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
    s[(row0 / g) * N + n] = reinterpret_cast<const uint16_t*>(wp + blob * blob_bytes + head)[u * kTileN + r];
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
        prepack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(s, N, KT, g, slots, ts, wp, blob, kCodeBytes);
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
        unpack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(wp, N, KT, g, slots, ts, s, blob, kCodeBytes);
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

// ------------------------------------------------------------------ 2:4 sparse weights
// One thread per (blob, code word w < 1024): w = (b*8 + rt)*32 + lane, lane = 4gc + t. The
// thread reads the four groups its word holds (groups t and t + 4 of columns 16rt + gc and
// + 8), picks each group's kept rows, writes the word and ORs its metadata nibbles with those
// of the quad's other lanes (t = 0..3), whose lanes 0 and 1 write the quad's two metadata
// words. A group with more than two codes other than 8 sets *bad (its two lowest such codes
// are kept). Launched in blocks of 256 over whole blobs, so a quad is always one warp's.
__global__ void prepack_sp24_codes_kernel(const uint32_t* __restrict__ Q, int N, int KT, long long total,
                                          uint8_t* __restrict__ wp, size_t blob_bytes, int* __restrict__ bad) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;  // total is a multiple of 1024: whole warps leave together
    const int w = static_cast<int>(idx % 1024);
    const long long blob = idx / 1024;
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const int b = w >> 8, rt = (w >> 5) & 7, gc = (w >> 2) & 7, t = w & 3;
    uint32_t code = 0, meta[2] = {0u, 0u};
    bool over = false;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const long long n = nt * kTileN + 16 * rt + 8 * half + gc;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int j = t + 4 * x;                                                // group: rows 32b + 4j ..
            const long long qrow = static_cast<long long>(kt) * 16 + 4 * b + (j >> 1);  // row of Q (8 codes)
            const uint32_t src = (n < N) ? __ldg(Q + qrow * N + n) : 0x88888888u;
            const uint32_t c4 = (src >> (16 * (j & 1))) & 0xFFFFu;  // the group's codes, position p at bits 4p
            uint32_t nz = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) nz |= (((c4 >> (4 * p)) & 0xFu) != 8u ? 1u : 0u) << p;
            over = over || __popc(nz) > 2;
            uint32_t keep = nz;
#pragma unroll
            for (int p = 0; p < 4; ++p)  // made up to two with the lowest rows of code 8
                if (__popc(keep) < 2 && !((keep >> p) & 1u)) keep |= 1u << p;
            const int p0 = __ffs(keep) - 1;
            const int p1 = __ffs(keep & (keep - 1)) - 1;
            code |= ((c4 >> (4 * p0)) & 0xFu) << (4 * (half + 2 * x));
            code |= ((c4 >> (4 * p1)) & 0xFu) << (4 * (half + 2 * x + 4));
            meta[x] |= static_cast<uint32_t>(p0 | (p1 << 2)) << (4 * (t + 4 * half));
        }
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        meta[x] |= __shfl_xor_sync(0xffffffffu, meta[x], 1);
        meta[x] |= __shfl_xor_sync(0xffffffffu, meta[x], 2);
    }
    uint8_t* base = wp + blob * blob_bytes;
    reinterpret_cast<uint32_t*>(base)[w] = code;
    if (t < 2) reinterpret_cast<uint32_t*>(base + kSpCodeBytes)[((b * 8 + rt) * 8 + gc) * 2 + t] = meta[t];
    if (over) *bad = 1;
}

// One thread per (blob, row i of Q within the k-block (8 codes), column r): rebuilds the 8
// codes (pruned rows as 8) from the code and metadata words of their two groups.
__global__ void unpack_sp24_codes_kernel(const uint8_t* __restrict__ wp, int N, int KT, long long total,
                                         uint32_t* __restrict__ Q, size_t blob_bytes) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int i = static_cast<int>((idx / kTileN) % 16);
    const long long blob = idx / (16 * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    if (n >= N) return;
    const uint8_t* base = wp + blob * blob_bytes;
    const uint32_t* code = reinterpret_cast<const uint32_t*>(base);
    const uint32_t* meta = reinterpret_cast<const uint32_t*>(base + kSpCodeBytes);
    const int b = i >> 2, rt = r >> 4, half = (r >> 3) & 1, gc = r & 7;
    uint32_t out = 0x88888888u;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int j = 2 * (i & 3) + e;  // group j: rows 32b + 4j .. = codes 4e .. 4e + 3 of this Q word
        const uint32_t m = (meta[((b * 8 + rt) * 8 + gc) * 2 + (j >> 2)] >> (4 * ((j & 3) + 4 * half))) & 0xFu;
        const uint32_t cw = code[(b * 8 + rt) * 32 + 4 * gc + (j & 3)];
        const int p0 = static_cast<int>(m & 3u), p1 = static_cast<int>(m >> 2);
        const uint32_t c0 = (cw >> (4 * (half + 2 * (j >> 2)))) & 0xFu;
        const uint32_t c1 = (cw >> (4 * (half + 2 * (j >> 2) + 4))) & 0xFu;
        out = (out & ~(0xFu << (4 * (4 * e + p0)))) | (c0 << (4 * (4 * e + p0)));
        out = (out & ~(0xFu << (4 * (4 * e + p1)))) | (c1 << (4 * (4 * e + p1)));
    }
    Q[(static_cast<long long>(kt) * 16 + i) * N + n] = out;
}

int launch_prepack_sp24(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, int* bad,
                        cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    const size_t blob = blob_bytes_sp24(slots > 0 ? slots : 0);
    uint8_t* wp = static_cast<uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 1024;
    prepack_sp24_codes_kernel<<<blocks_for(tc, 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(Q), N, KT, tc,
                                                                    wp, blob, bad);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        prepack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(s, N, KT, g, slots, ts, wp, blob, kSpHeadBytes);
    } else {
        const int tail_elems = static_cast<int>(channel_tail_bytes(N) / 2);
        channel_tail_kernel<<<blocks_for(tail_elems, 256), 256, 0, st>>>(
            s, N, NT * kTileN, tail_elems, reinterpret_cast<uint16_t*>(wp + nblob * blob));
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_unpack_sp24(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    const size_t blob = blob_bytes_sp24(slots > 0 ? slots : 0);
    const uint8_t* wp = static_cast<const uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 16 * kTileN;
    unpack_sp24_codes_kernel<<<blocks_for(tc, 256), 256, 0, st>>>(wp, N, KT, tc, reinterpret_cast<uint32_t*>(Q), blob);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        unpack_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(wp, N, KT, g, slots, ts, s, blob, kSpHeadBytes);
    } else {
        channel_untail_kernel<<<blocks_for(N, 256), 256, 0, st>>>(
            reinterpret_cast<const uint16_t*>(wp + nblob * blob), N, s);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// ------------------------------------------------------------------ mixed 2/4-bit weights
// The blob table at the start of the buffer is written by the host first (offsets are a
// prefix sum over the widths); these kernels read it for each blob's offset and widths.
__device__ __forceinline__ int mixed_block_offset(uint32_t wbits, int v) {
    return kMixBlock2 * (v + __popc(wbits & ((1u << v) - 1u)));
}

// 2-bit field of row 8t + r of column 16rt + gc + 8j within the word of lane (gc, t).
__device__ __forceinline__ int mixed_field(int r, int j) { return (r >> 1) + 4 * j + 8 * (r & 1); }

// One thread per (blob, block v, r < 128). A 4-bit block: the four words of column r, as in a
// W4A16 blob. A 2-bit block: words r and r + 128 of the block (word w = rt*32 + 4gc + t covers
// columns 16rt + gc and + 8, rows 8t .. 8t + 7). A code above 3 in a 2-bit block sets *bad.
// Padded columns hold the block's zero point (8 or 2): weight 0.
__global__ void prepack_mixed_codes_kernel(const uint32_t* __restrict__ Q, int N, int KT, long long total,
                                           uint8_t* __restrict__ wp, int* __restrict__ bad) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int v = static_cast<int>((idx / kTileN) % 4);
    const long long blob = idx / (4 * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const uint32_t e = reinterpret_cast<const uint32_t*>(wp)[blob];
    uint8_t* block = wp + static_cast<size_t>(e >> 4) * 16 + mixed_block_offset(e & 0xFu, v);
    if ((e >> v) & 1u) {
        const long long n = nt * kTileN + r;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const long long row = static_cast<long long>(kt) * 16 + v * 4 + i;  // row of Q (8 codes)
            w[i] = (n < N) ? permute_word<false>(__ldg(Q + row * N + n)) : 0x88888888u;
        }
        *reinterpret_cast<uint4*>(block + static_cast<size_t>(r) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        return;
    }
    bool over = false;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int wi = r + h * kTileN;
        const int rt = wi >> 5, gc = (wi >> 2) & 7, t = wi & 3;
        const long long row = static_cast<long long>(kt) * 16 + v * 4 + t;  // rows 32v + 8t .. + 7
        uint32_t out = 0;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const long long n = nt * kTileN + 16 * rt + gc + 8 * j;
            const uint32_t src = (n < N) ? __ldg(Q + row * N + n) : 0x22222222u;
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                const uint32_t c = (src >> (4 * rr)) & 0xFu;
                over = over || c > 3u;
                out |= (c & 3u) << (2 * mixed_field(rr, j));
            }
        }
        reinterpret_cast<uint32_t*>(block)[wi] = out;
    }
    if (over) *bad = 1;
}

// One thread per (blob, slot, r): the group scale of column r after the blob's code blocks.
__global__ void prepack_mixed_scales_kernel(const uint16_t* __restrict__ s, int N, int KT, int g, int slots,
                                            long long total, uint8_t* __restrict__ wp) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const uint32_t e = reinterpret_cast<const uint32_t*>(wp)[blob];
    const long long grp = (static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g) / g;
    uint16_t* sc = reinterpret_cast<uint16_t*>(wp + static_cast<size_t>(e >> 4) * 16 + mixed_block_offset(e & 0xFu, 4));
    sc[u * kTileN + r] = (n < N) ? s[grp * N + n] : static_cast<uint16_t>(0);
}

// Inverse (a test aid): one thread per (blob, block v, r): the Q words of column r in block v and
// (r == 0) the block's width.
__global__ void unpack_mixed_codes_kernel(const uint8_t* __restrict__ wp, int N, int KT, int NT, long long total,
                                          uint32_t* __restrict__ Q, uint8_t* __restrict__ widths) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int v = static_cast<int>((idx / kTileN) % 4);
    const long long blob = idx / (4 * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const uint32_t e = reinterpret_cast<const uint32_t*>(wp)[blob];
    const bool four = (e >> v) & 1u;
    if (r == 0) widths[(static_cast<long long>(kt) * 4 + v) * NT + nt] = four ? 4 : 2;
    const long long n = nt * kTileN + r;
    if (n >= N) return;
    const uint8_t* block = wp + static_cast<size_t>(e >> 4) * 16 + mixed_block_offset(e & 0xFu, v);
    const int rt = r >> 4, j = (r >> 3) & 1, gc = r & 7;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t out;
        if (four) {
            out = unpermute_word<false>(reinterpret_cast<const uint32_t*>(block)[r * 4 + i]);
        } else {
            const uint32_t x = reinterpret_cast<const uint32_t*>(block)[rt * 32 + 4 * gc + i];
            out = 0;
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) out |= ((x >> (2 * mixed_field(rr, j))) & 3u) << (4 * rr);
        }
        Q[(static_cast<long long>(kt) * 16 + v * 4 + i) * N + n] = out;
    }
}

__global__ void unpack_mixed_scales_kernel(const uint8_t* __restrict__ wp, int N, int KT, int g, int slots,
                                           long long total, uint16_t* __restrict__ s) {
    const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (idx >= total) return;
    const int r = static_cast<int>(idx % kTileN);
    const int u = static_cast<int>((idx / kTileN) % slots);
    const long long blob = idx / (static_cast<long long>(slots) * kTileN);
    const int kt = static_cast<int>(blob % KT);
    const long long nt = blob / KT;
    const long long n = nt * kTileN + r;
    const long long row0 = static_cast<long long>(kt) * kTileK + static_cast<long long>(u) * g;
    if (n >= N || row0 % g != 0) return;
    const uint32_t e = reinterpret_cast<const uint32_t*>(wp)[blob];
    s[(row0 / g) * N + n] = reinterpret_cast<const uint16_t*>(
        wp + static_cast<size_t>(e >> 4) * 16 + mixed_block_offset(e & 0xFu, 4))[u * kTileN + r];
}

int launch_prepack_mixed(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, int* bad,
                         cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    uint8_t* wp = static_cast<uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 4 * kTileN;
    prepack_mixed_codes_kernel<<<blocks_for(tc, 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(Q), N, KT, tc,
                                                                     wp, bad);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        prepack_mixed_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(s, N, KT, g, slots, ts, wp);
    } else {
        const int tail_elems = static_cast<int>(channel_tail_bytes(N) / 2);
        channel_tail_kernel<<<blocks_for(tail_elems, 256), 256, 0, st>>>(
            s, N, NT * kTileN, tail_elems, reinterpret_cast<uint16_t*>(wp + mixed_table_bytes(nblob)));
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_unpack_mixed(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, uint8_t* widths,
                        cudaStream_t st) {
    const int slots = scale_slots(K, g);
    const int KT = K / kTileK, NT = n_tiles(N);
    const uint8_t* wp = static_cast<const uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(NT) * KT;
    const long long tc = nblob * 4 * kTileN;
    unpack_mixed_codes_kernel<<<blocks_for(tc, 256), 256, 0, st>>>(wp, N, KT, NT, tc, reinterpret_cast<uint32_t*>(Q),
                                                                    widths);
    if (slots > 0) {
        const long long ts = nblob * slots * kTileN;
        unpack_mixed_scales_kernel<<<blocks_for(ts, 256), 256, 0, st>>>(wp, N, KT, g, slots, ts, s);
    } else {
        channel_untail_kernel<<<blocks_for(N, 256), 256, 0, st>>>(
            reinterpret_cast<const uint16_t*>(wp + mixed_table_bytes(nblob)), N, s);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wq
