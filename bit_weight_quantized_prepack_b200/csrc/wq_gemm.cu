// The mixed-precision linear layer on sm_100a: Y[M,N] = A[M,K] . dequant(Wp).
//
// What the pages ask of it ("MARLIN: Mixed-Precision Auto-Regressive Parallel Inference on
// Large Language Models", Abstract): stay memory-bound on the 4-bit weights over batch
// sizes 1..128 through asynchronous memory access, task scheduling, pipelining and bespoke
// quantisation support; hide the dequantisation ("Enabling Fast 2-bit LLM on GPUs: Memory
// Alignment and Asynchronous Dequantization", Abstract: dequantisation otherwise takes more
// than half of the run time). How these kernels do it on B200 (three families, picked by the
// number of activation rows M; all share the prepacked layout, the stream-K walk, the producers
// and the shared-memory ring):
//
//   * M <= 16: the register-operand kernel (wq_gemm_rf, at the end of this file): every warp
//     dequantises its share of each k-block into registers and multiplies it with the
//     warp-level MMA (mma.sync), no tensor memory and no hand-off between warps. At so few rows
//     the tensor-memory chain below costs more per k-block than the arithmetic.
//   * M = 17..32 (small tiles) and M > 32 (large tiles): the tcgen05 kernels described next.
//     The weights are the MMA's M operand (128 output columns per tile) and the activations
//     its N operand (tile_m rows, 32..256).
//   * One persistent CTA per SM walks a contiguous range of (tile, k-block) units (stream-K).
//     A tile split between CTAs is finished by the CTA holding its last k-block, which adds
//     the other CTAs' partial sums in a fixed order: results are deterministic.
//   * Warp roles per CTA of the tcgen05 kernels (704 threads in both designs):
//       warp 20     weight producer: one bulk copy moves up to 4 consecutive blobs (codes +
//                   scales of 4 k-blocks, contiguous in HBM by construction of the prepack);
//       warp 21     activation producer: one 3-D tensor copy moves the same k-blocks of the
//                   activation tile (128-byte swizzle, the MMA's K-major B layout);
//       warps 0..15 dequantisation: each thread owns one weight column of the tile (one
//                   tensor-memory lane); it turns packed words into fp16 (or int8) values in
//                   registers and stores them into tensor memory, where they are the MMA's A
//                   operand: the dequantised weights never touch shared memory. The walk's
//                   k-blocks are dealt round-robin to groups of these warps, so that several
//                   k-blocks per lane quarter are in flight at once;
//       warps 16..19 MMA issuers (one elected thread each).
//     Two ways to split the work, by tile height:
//       small tiles (tile_m = 32): 4 residues; issuer r owns
//                   every fourth k-block and writes each k-block's product into a fresh
//                   partial in tensor memory (two buffers per residue, used in turn), which
//                   the dequant warps of residue r add in fp32 registers (applying the group
//                   scale there, acc += s * P, for g >= 128, so the dequant emits exact q - 8)
//                   while the MMAs of the next k-block run; the four residues combine at
//                   each segment's end and run the epilogue;
//       large tiles: 2 residues of 8 dequant warps (4 lane quarters x 2 halves of a
//                   k-block); issuer q owns a quarter (or half, or all) of every k-block's K
//                   range and accumulates the whole segment in tensor memory; the dequant
//                   applies the scale and the dequant warps run the epilogue.
//     Measured on B200: a thread issuing tcgen05.mma back to back gets one instruction per
//     ~75-85 cycles whatever the shape, and one issuing bulk copies gets one copy per ~270 ns;
//     several issuing warps and copies of 16-33 KB take both costs off the critical path.
//     At small M each residue's k-block is a chain (dequant into the A slot, MMA issue,
//     completion, next dequant) whose length, with four chains per SM, sets the ceiling: the
//     reason the register-operand kernel takes M <= 16.
//   * Every wait is bounded by a global-timer limit; an expired wait records WQ_ERR_TIMEOUT
//     and the CTA winds down (drains its copies and MMAs, frees tensor memory) instead of
//     hanging.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "wq.h"
#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {

struct Barriers {
    uint64_t full[kChunkBars];     // chunk landed: both producers' bytes (count 2 + transactions),
                                   // indexed by chunk sequence number mod kChunkBars
    uint64_t empty_w[kMaxSlots];   // weight slot read by the 8 dequant warps
    uint64_t empty_a[kMaxSlots];   // activation slot read by the MMAs of every issuer (commits)
    uint64_t afull[kASlotsS][2];   // dequantised k-block (half) in tensor memory (4 warps each)
    uint64_t aempty[kASlotsS];     // MMAs done with a tensor-memory slot
    uint64_t dfull;                // accumulators of a segment complete (one commit per issuer)
    uint64_t drain[kMaxIssuers];   // all MMAs of an issuer complete
    uint32_t wbits[kMaxSlots];     // mixed 2/4-bit: the widths of the blob in each weight slot
    uint64_t tbl_full;             // mixed 2/4-bit: the CTA's table entries landed in shared memory
};

struct Ctl {
    volatile int* abort_flag;      // shared: set by the first wait that gives up
    int* status;
    unsigned long long timeout_ns;
};

// Modes with group scales in the blob (symmetric, or with a zero point per group).
__host__ __device__ constexpr bool is_group(int mode) { return mode == kModeGroup || mode == kModeGroupZP; }

__device__ __forceinline__ void raise_error(const Ctl& c, int code) {
    *c.abort_flag = 1;
    atomicCAS(c.status, 0, code);
}

// Bounded wait on an mbarrier phase. Returns false when the CTA aborts or the limit expires.
// The common case (phase already complete) is one inline non-blocking test; otherwise each
// poll lets the thread sleep in hardware until the phase completes (up to 20 us), so waiting
// warps do not take issue slots or ALU cycles from the dequantising warps.
__device__ __forceinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, const Ctl& c, bool honour_abort) {
    constexpr uint32_t kSuspendNs = 20000;
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
        if (honour_abort && *c.abort_flag) return false;
        if (global_timer_ns() - t0 > c.timeout_ns) {
            raise_error(c, WQ_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c, bool honour_abort = true) {
    if (mbar_test_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, c, honour_abort);
}

// Bounded wait for a stream-K publish flag written by another CTA.
__device__ bool wait_flag(const int* flag, const Ctl& c) {
    if (ld_acquire_gpu(flag) != 0) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (ld_acquire_gpu(flag) != 0) return true;
        if (*c.abort_flag) return false;
        if (global_timer_ns() - t0 > c.timeout_ns) {
            raise_error(c, WQ_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
}

// First unit of CTA c under the even split of `units` over `grid` CTAs.
__device__ __forceinline__ long long unit_start(int c, long long units, int grid) {
    return static_cast<long long>(c) * units / grid;
}

// Walks a CTA's unit range [beg, end) one segment (a run of k-blocks of one tile) at a time,
// last segment first. Going backwards makes the CTA holding a tile's last k-block, which
// finishes the tile, reach that tile last, while the CTAs it waits for have lower indices
// and reach their part of the tile first. Inside a segment the k-blocks go forward, so the
// blobs of a chunk are contiguous in HBM and in the shared-memory ring.
struct SegCursor {
    long long it, beg;
    int k_blocks;
    int tile, kb_hi, kb_lo;
    bool owner, whole;
    __device__ SegCursor(long long b, long long e, int kbs) : it(e - 1), beg(b), k_blocks(kbs) {}
    __device__ bool next() {
        if (it < beg) return false;
        tile = static_cast<int>(it / k_blocks);
        const long long tbase = static_cast<long long>(tile) * k_blocks;
        const long long lo = beg > tbase ? beg : tbase;
        kb_hi = static_cast<int>(it - tbase);
        kb_lo = static_cast<int>(lo - tbase);
        owner = kb_hi == k_blocks - 1;
        whole = owner && kb_lo == 0;
        it = lo - 1;
        return true;
    }
};

// Length of the chunk that starts at k-block kb of a segment ending at kb_hi, at ring slot pos:
// at most `chunk` k-blocks, never past the segment, never wrapping the ring. The CTA's first
// chunk (first: walk index 0) is one k-block: every CTA asks for its first chunk at the same
// moment, when the grid dependency resolves, and the smaller it is the sooner the consumers
// start (the rest streams in behind it).
__device__ __forceinline__ int chunk_len(int chunk, int kb, int kb_hi, int pos, int slots, bool first) {
    int c = kb_hi - kb + 1;
    if (c > chunk) c = chunk;
    if (c > slots - pos) c = slots - pos;
    if (first && c > 1) c = 1;
    return c;
}

// The full barrier of chunk number ch (counted along the CTA's walk) is full[ch % kChunkBars]
// and the chunk completes that barrier's phase ch / kChunkBars. With more barriers than ring
// slots, a barrier is re-armed only after the ring has moved past every slot of the chunk that
// last used it, so a role that still holds one of that chunk's k-blocks can never see the
// barrier two phases ahead (a slot-indexed barrier could, when chunk boundaries shift).
__device__ __forceinline__ uint32_t chunk_bar(uint32_t ch) { return ch % kChunkBars; }
__device__ __forceinline__ uint32_t chunk_parity(uint32_t ch) { return (ch / kChunkBars) & 1u; }

// The same two numbers kept incrementally along the walk (no division per chunk).
struct ChunkBar {
    uint32_t bar = 0, parity = 0;
    __device__ __forceinline__ void next() {
        if (++bar == static_cast<uint32_t>(kChunkBars)) {
            bar = 0;
            parity ^= 1u;
        }
    }
};

// ------------------------------------------------------------------ dequantisation
// fp16 constants from the binary16 format: 0x6400 = 1024 (exponent field 25, so the 10
// mantissa bits count units), 0x6408 = 1032 = 1024 + 8, 0x2C00 = 1/16, 0xD480 = -72.
// (w & 0x000F000F) | 0x64006400 is the fp16 pair (1024 + q_lo, 1024 + q_hi) exactly;
// subtracting 1032 leaves q - 8 exactly. A nibble in bits 4..7 of a half gives 1024 + 16q;
// (1024 + 16q)/16 - 72 = q - 8, again exact in one fused multiply-add.
// With a zero point z per group (asymmetric groups) the two constants become 1024 + z and
// -(64 + z): (1024 + q) - (1024 + z) and (1024 + 16q)/16 - (64 + z) are q - z, exact.
__device__ __forceinline__ __half2 half2_bits(uint32_t v) { return *reinterpret_cast<const __half2*>(&v); }
// The constants of zero point z (0..15): 0x6400 + z is 1024 + z (units of 1 in [1024, 2048)),
// 0xD400 + 16z is -(64 + z) (units of 1/16 in [64, 128)).
__device__ __forceinline__ uint32_t zp_lo(uint32_t z) { return (0x6400u + z) * 0x10001u; }
__device__ __forceinline__ uint32_t zp_hi(uint32_t z) { return (0xD400u + (z << 4)) * 0x10001u; }

__device__ __forceinline__ void dequant_word_f16(uint32_t x, __half2 s, bool scaled, uint32_t* out) {
    const uint32_t kMagic = 0x64006400u;
    const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
    const __half2 kSixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    const __half2 kMinus72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
    const uint32_t x8 = x >> 8;
    const uint32_t u0 = lop3_and_or(x, 0x000F000Fu, kMagic);
    const uint32_t u1 = lop3_and_or(x, 0x00F000F0u, kMagic);
    const uint32_t u2 = lop3_and_or(x8, 0x000F000Fu, kMagic);
    const uint32_t u3 = lop3_and_or(x8, 0x00F000F0u, kMagic);
    __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&u0), k1032);
    __half2 h1 = __hfma2(*reinterpret_cast<const __half2*>(&u1), kSixteenth, kMinus72);
    __half2 h2 = __hsub2(*reinterpret_cast<const __half2*>(&u2), k1032);
    __half2 h3 = __hfma2(*reinterpret_cast<const __half2*>(&u3), kSixteenth, kMinus72);
    if (scaled) {  // one round-to-nearest of (q - 8) * s per weight
        h0 = __hmul2(h0, s);
        h1 = __hmul2(h1, s);
        h2 = __hmul2(h2, s);
        h3 = __hmul2(h3, s);
    }
    out[0] = *reinterpret_cast<uint32_t*>(&h0);
    out[1] = *reinterpret_cast<uint32_t*>(&h1);
    out[2] = *reinterpret_cast<uint32_t*>(&h2);
    out[3] = *reinterpret_cast<uint32_t*>(&h3);
}

// The same with the zero point's constants klo = zp_lo(z), khi = zp_hi(z): q - z exactly.
__device__ __forceinline__ void dequant_word_f16_zp(uint32_t x, __half2 s, bool scaled, uint32_t klo, uint32_t khi,
                                                    uint32_t* out) {
    const uint32_t kMagic = 0x64006400u;
    const __half2 kSixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    const uint32_t x8 = x >> 8;
    const uint32_t u0 = lop3_and_or(x, 0x000F000Fu, kMagic);
    const uint32_t u1 = lop3_and_or(x, 0x00F000F0u, kMagic);
    const uint32_t u2 = lop3_and_or(x8, 0x000F000Fu, kMagic);
    const uint32_t u3 = lop3_and_or(x8, 0x00F000F0u, kMagic);
    __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&u0), half2_bits(klo));
    __half2 h1 = __hfma2(*reinterpret_cast<const __half2*>(&u1), kSixteenth, half2_bits(khi));
    __half2 h2 = __hsub2(*reinterpret_cast<const __half2*>(&u2), half2_bits(klo));
    __half2 h3 = __hfma2(*reinterpret_cast<const __half2*>(&u3), kSixteenth, half2_bits(khi));
    if (scaled) {
        h0 = __hmul2(h0, s);
        h1 = __hmul2(h1, s);
        h2 = __hmul2(h2, s);
        h3 = __hmul2(h3, s);
    }
    out[0] = *reinterpret_cast<uint32_t*>(&h0);
    out[1] = *reinterpret_cast<uint32_t*>(&h1);
    out[2] = *reinterpret_cast<uint32_t*>(&h2);
    out[3] = *reinterpret_cast<uint32_t*>(&h3);
}

// int8 lanes 16*(q - 8): the code moved to the high nibble of its byte with the sign bit
// flipped ((q ^ 8) << 4) is 16*(q - 8) in two's complement. The accumulator is shifted
// right by 4 in the epilogue, exactly.
__device__ __forceinline__ void dequant_word_i8(uint32_t x, uint32_t* out) {
    out[0] = lop3_and_xor(x << 4, 0xF0F0F0F0u, 0x80808080u);  // codes 0..3 (low nibbles)
    out[1] = lop3_and_xor(x, 0xF0F0F0F0u, 0x80808080u);       // codes 4..7 (high nibbles)
}

// ------------------------------------------------------------------ epilogue
// Sum of the issuers' accumulators for 8 columns (fixed order), as raw 32-bit values.
template <int MODE>
__device__ __forceinline__ void load_acc8(uint32_t taddr, int issuers, int tile_m, uint32_t* v) {
    tmem_ld_x8(taddr, v);
    for (int q = 1; q < issuers; ++q) {
        uint32_t w[8];
        tmem_ld_x8(taddr + static_cast<uint32_t>(q * tile_m), w);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (MODE == kModeW4A8)
                v[j] = static_cast<uint32_t>(static_cast<int32_t>(v[j]) + static_cast<int32_t>(w[j]));
            else
                v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(w[j]));
        }
    }
    tmem_ld_wait();
}

template <int MODE>
__device__ void epilogue(const GemmArgs& p, Barriers& b, uint32_t tmem, const Ctl& ctl, const SegCursor& seg,
                         int seg_index, int part, int quarter, int lane) {
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int nt = seg.tile / p.m_tiles, mt = seg.tile % p.m_tiles;
    const int n = nt * kTileN + row;
    // the 4 dequant warps of a lane quarter split the tile rows in runs of a multiple of 8
    // (tile_m is a multiple of 16, so every run is too; the last may be short or empty)
    const int cols_per = ((p.tile_m / 4 + 7) / 8) * 8;
    const int c_begin = part * cols_per;
    int cols = p.tile_m - c_begin;
    cols = cols < 0 ? 0 : (cols > cols_per ? cols_per : cols);
    const int m_base = mt * p.tile_m + c_begin;

    bool ok = __all_sync(0xffffffffu, wait_bar(&b.dfull, seg_index & 1, ctl));
    tc_fence_after();

    if (!seg.owner) {
        // contributor: publish this CTA's fp32 (or int32) partial tile, then raise its flag
        uint32_t* part = reinterpret_cast<uint32_t*>(p.ws_partial) + static_cast<size_t>(blockIdx.x) * p.tile_m * kTileN;
        for (int c = 0; c < cols; c += 8) {
            uint32_t v[8];
            if (ok) {
                load_acc8<MODE>(tmem + lane_base + static_cast<uint32_t>(c_begin + c), p.issuers, p.tile_m, v);
#pragma unroll
                for (int j = 0; j < 8; ++j) part[static_cast<size_t>(c_begin + c + j) * kTileN + row] = v[j];
            }
        }
        // the barrier orders every thread's partial stores before the leader's release of the flag
        // (the release is cumulative), so no thread needs a GPU-scope fence of its own
        tc_fence_before();
        named_barrier_sync(1, kNumDqWarps * 32);  // also: every warp has read the accumulators
        if (threadIdx.x == 0 && ok && !*ctl.abort_flag && static_cast<int>(blockIdx.x) != p.skip_publish)
            st_release_gpu(&p.ws_flags[blockIdx.x], 1);
        return;
    }

    // owner: the contributing CTAs are those before it whose unit range reaches into the tile
    // (closed form: the CTA holding the tile's first unit is the smallest c with
    // unit_start(c + 1) > tbase); each lane polls one contributor's flag
    const int me = static_cast<int>(blockIdx.x);
    int c_last = me;  // contributors are CTAs c_last .. me - 1
    if (!seg.whole) {
        const long long tbase = static_cast<long long>(seg.tile) * p.k_blocks;
        c_last = static_cast<int>(((tbase + 1) * p.grid + p.units - 1) / p.units) - 1;
        const int ncontrib = me - c_last;
        for (int j0 = 0; j0 < ncontrib; j0 += 32) {
            bool good = true;
            if (ok && j0 + lane < ncontrib) good = wait_flag(&p.ws_flags[me - 1 - j0 - lane], ctl);
            ok = __all_sync(0xffffffffu, good) && ok;
        }
        __syncwarp();  // the polling lanes' acquires order the whole warp's loads below
    }

    float s_col = 1.0f;
    if (MODE == kModeChannel) s_col = __half2float(__ushort_as_half(p.s_chan[n]));
    float sw_col = 0.0f;
    if (MODE == kModeW4A8) sw_col = n < p.N ? p.sw[n] : 0.0f;

    // 16 columns at a time: the 16 loads of a contributor's partial are in flight together
    for (int c = 0; c < cols && ok; c += 16) {
        uint32_t v[16];
        const bool two = c + 8 < cols;
        load_acc8<MODE>(tmem + lane_base + static_cast<uint32_t>(c_begin + c), p.issuers, p.tile_m, v);
        if (two) load_acc8<MODE>(tmem + lane_base + static_cast<uint32_t>(c_begin + c + 8), p.issuers, p.tile_m, v + 8);
        for (int cc = me - 1; cc >= c_last; --cc) {
            const uint32_t* part =
                reinterpret_cast<const uint32_t*>(p.ws_partial) + static_cast<size_t>(cc) * p.tile_m * kTileN;
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                w[j] = (j < 8 || two) ? __ldcg(part + static_cast<size_t>(c_begin + c + j) * kTileN + row) : 0u;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (MODE == kModeW4A8)
                    v[j] = static_cast<uint32_t>(static_cast<int32_t>(v[j]) + static_cast<int32_t>(w[j]));
                else
                    v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(w[j]));
            }
        }
        if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int m = m_base + c + j;
                if ((j < 8 || two) && m < p.M) {
                    const size_t o = static_cast<size_t>(m) * p.N + n;
                    float y;
                    if (MODE == kModeW4A8) {
                        const int32_t acc = static_cast<int32_t>(v[j]) >> 4;
                        if (p.acc_out) p.acc_out[o] = acc;
                        const float t = static_cast<float>(acc) * p.sa[m];
                        y = t * sw_col;
                    } else if (MODE == kModeChannel) {
                        y = __uint_as_float(v[j]) * s_col;
                    } else {
                        y = __uint_as_float(v[j]);
                    }
                    p.y[o] = __half_as_ushort(__float2half_rn(y));
                }
            }
        }
    }
    // every dequant warp has read the accumulators (and the partials): only then may one of
    // them hand the next segment's first k-block to the MMA, which overwrites the accumulators
    tc_fence_before();
    named_barrier_sync(1, kNumDqWarps * 32);
    // ready for the next call, but only when every wait of the CTA succeeded: after an expired
    // wait a contributor may still publish late, and the flags stay set until the host clears
    // them (wq_get_device_status)
    if (!seg.whole && threadIdx.x == 0 && !*ctl.abort_flag)
        for (int cc = me - 1; cc >= c_last; --cc) p.ws_flags[cc] = 0;
}

// ------------------------------------------------------------------ roles
template <int MODE>
__device__ void dequant_role(const GemmArgs& p, const uint8_t* wring, Barriers& b, uint32_t tmem, const Ctl& ctl,
                             long long beg, long long end) {
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;  // 128 k of fp16 or int8 per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, half = (warp >> 2) & 1;
    const uint32_t residue = static_cast<uint32_t>(warp >> 3);  // this group's k-blocks: walk index mod 2
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int u0 = (64 * half) / p.group_rows, u1 = (64 * half + 32) / p.group_rows;
    ChunkBar cb;
    uint32_t iter = 0;
    int pos = 0, seg_index = 0;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, iter == 0);
            const uint32_t fb = cb.bar, fpar = cb.parity;
            cb.next();
            const bool mine = ((residue + kDqResidues - iter % kDqResidues) % kDqResidues) < static_cast<uint32_t>(c);
            bool ok = !mine || __all_sync(0xffffffffu, wait_bar(&b.full[fb], fpar, ctl));
            for (int t = 0; t < c; ++t, ++iter) {
                if (iter % kDqResidues != residue) continue;
                const int s = pos + t;
                const uint32_t a = iter % kASlots, aph = (iter / kASlots) & 1;
                uint4 w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
                uint16_t sc0 = 0, sc1 = 0;
                uint32_t z0 = 8, z1 = 8;
                if (ok) {
                    const uint8_t* blob = wring + static_cast<size_t>(s) * p.blob_bytes;
                    const uint4* words = reinterpret_cast<const uint4*>(blob);
                    w0 = words[(half * 2 + 0) * kTileN + row];
                    w1 = words[(half * 2 + 1) * kTileN + row];
                    if (is_group(MODE) && p.scale_in_dequant) {
                        const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + kCodeBytes);
                        sc0 = sc[u0 * kTileN + row];
                        sc1 = sc[u1 * kTileN + row];
                    }
                    if (MODE == kModeGroupZP) {
                        z0 = blob[p.zp_offset + u0 * kTileN + row];
                        z1 = blob[p.zp_offset + u1 * kTileN + row];
                    }
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&b.empty_w[s]);
                if (ok) ok = __all_sync(0xffffffffu, wait_bar(&b.aempty[a], aph ^ 1, ctl));
                if (ok) {
                    const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    const uint32_t taddr = tmem + lane_base + kTmemAOffset + a * kSlotCols + half * (kSlotCols / 2);
                    if (MODE == kModeW4A8) {
                        uint32_t out[16];
#pragma unroll
                        for (int i = 0; i < 8; ++i) dequant_word_i8(wv[i], out + 2 * i);
                        tmem_st_x16(taddr, out);
                    } else {
                        uint32_t out[32];
                        const __half2 s0 = __half2half2(__ushort_as_half(sc0));
                        const __half2 s1 = __half2half2(__ushort_as_half(sc1));
                        if (MODE == kModeGroupZP) {
                            const uint32_t lo0 = zp_lo(z0), hi0 = zp_hi(z0), lo1 = zp_lo(z1), hi1 = zp_hi(z1);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dequant_word_f16_zp(wv[i], i < 4 ? s0 : s1, true, i < 4 ? lo0 : lo1, i < 4 ? hi0 : hi1,
                                                    out + 4 * i);
                        } else if (MODE == kModeGroup && p.scale_in_dequant) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) dequant_word_f16(wv[i], i < 4 ? s0 : s1, true, out + 4 * i);
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) dequant_word_f16(wv[i], s0, false, out + 4 * i);
                        }
                        tmem_st_x32(taddr, out);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&b.afull[a][half]);
            }
            kb += c;
            pos += c;
            if (pos == p.slots) pos = 0;
        }
        epilogue<MODE>(p, b, tmem, ctl, seg, seg_index, static_cast<int>(residue) * 2 + half, quarter, lane);
        ++seg_index;
    }
}

// Weight producer (kWeightWarp, one thread) or activation producer (kActWarp, one thread).
// Mixed 2/4-bit weights: the weight producer warp (all 32 lanes) copies the CTA's table entries
// (units beg .. end, entries tlo .. thi - 1 around them; a unit's index is its blob's index) into
// shared memory once, after the grid dependency, and checks every blob the CTA will copy: it lies
// inside the caller's buffer and has the size its widths imply. A table that does not describe
// the format stops the CTA with WQ_ERR_INVALID_ARG before any weight copy. Returns whether the
// producer may go on (the same on every lane).
__device__ bool mixed_table_window(const GemmArgs& p, Barriers& b, uint32_t* tbl, const Ctl& ctl, long long beg,
                                   long long end, int lane, long long* tlo_out) {
    griddep_wait();  // the table is caller memory a preceding kernel may still write
    const long long tlo = beg & ~3ll;
    const long long thi = (end + 1 + 3) & ~3ll;  // entries beg .. end, 16-byte aligned around them
    *tlo_out = tlo;
    if (lane == 0) {
        mbar_arrive_expect_tx(&b.tbl_full, static_cast<uint32_t>((thi - tlo) * 4));
        bulk_g2s(tbl, p.mix_table + tlo, static_cast<uint32_t>((thi - tlo) * 4), &b.tbl_full, l2_policy_evict_first());
    }
    const bool landed = __all_sync(0xffffffffu, wait_bar(&b.tbl_full, 0, ctl));
    if (!landed) return false;
    const unsigned long long scale_bytes = static_cast<unsigned long long>(p.blob_bytes - kCodeBytes);
    bool valid = true;
    for (long long u = beg + lane; u < end; u += 32) {
        const uint32_t e0 = tbl[u - tlo], e1 = tbl[u + 1 - tlo];
        const unsigned long long lo = (e0 >> 4) * 16ull, hi = (e1 >> 4) * 16ull;
        const unsigned long long want = static_cast<unsigned long long>(kMixBlock2) * (4 + __popc(e0 & 0xFu)) + scale_bytes;
        valid = valid && hi > lo && hi - lo == want && hi <= p.wp_bytes;
    }
    valid = __all_sync(0xffffffffu, valid);
    if (!valid && lane == 0) raise_error(ctl, WQ_ERR_INVALID_ARG);
    return valid;
}

// kMix (mixed 2/4-bit weights, weight producer): tbl holds the CTA's table entries from entry
// tlo on, checked by mixed_table_window (tbl_ok).
template <int MODE, bool kWeights, bool kMix = false>
__device__ void producer_role(const ActMaps* maps, const GemmArgs& p, uint8_t* aring, uint8_t* wring, Barriers& b,
                              const Ctl& ctl, long long beg, long long end, const uint32_t* tbl = nullptr,
                              long long tlo_in = 0, bool tbl_ok = true) {
    const uint64_t policy = l2_policy_evict_first();  // every weight byte is read once
    uint32_t ebits = 0, ch = 0, armed = 0;
    ChunkBar cb;
    uint32_t first_pass_chunks = 0xffffffffu;  // chunks before the ring first wraps
    int pos = 0;
    bool ok = true;
    // A preceding kernel of the stream may still be writing the activations or the prepacked
    // weights: nothing is copied before it has completed. Everything else in the CTA that
    // reads or writes memory shared with it (the partials, flags and Y) comes after these
    // copies.
    griddep_wait();
    const long long tlo = tlo_in;  // kMix: first table entry held in tbl (a multiple of 4 entries)
    if (kWeights && kMix) ok = tbl_ok;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        const int nt = seg.tile / p.m_tiles, mt = seg.tile % p.m_tiles;
        const uint8_t* wtile = p.wp + static_cast<size_t>(nt) * p.k_blocks * p.blob_bytes;
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, ch == 0);
            for (int t = 0; t < c; ++t) {
                const int s = pos + t;
                if (ok && ch >= first_pass_chunks)  // a slot's first use needs no wait
                    ok = wait_bar(kWeights ? &b.empty_w[s] : &b.empty_a[s], ((ebits >> s) & 1u) ^ 1u, ctl);
                ebits ^= 1u << s;
            }
            if (ok) {
                uint64_t* fbar = &b.full[cb.bar];
                if (kWeights && kMix) {
                    // blobs of varying size: offsets and widths from the CTA's table entries (checked
                    // once, before the walk), one copy per blob into its fixed-stride slot; the
                    // widths reach the consumers through the slot's word, ordered before them by
                    // this thread's arrival (release)
                    const uint32_t* te = tbl + (static_cast<long long>(nt) * p.k_blocks + kb - tlo);
                    uint32_t e[kMaxChunk + 1];
#pragma unroll
                    for (int t = 0; t <= kMaxChunk; ++t) e[t] = (t <= c) ? te[t] : 0u;
                    uint32_t bytes = 0;
#pragma unroll
                    for (int t = 0; t < kMaxChunk; ++t)
                        if (t < c) {
                            b.wbits[pos + t] = e[t] & 0xFu;
                            bytes += ((e[t + 1] >> 4) - (e[t] >> 4)) * 16u;
                        }
                    mbar_arrive_expect_tx(fbar, bytes);
#pragma unroll
                    for (int t = 0; t < kMaxChunk; ++t)
                        if (t < c)
                            bulk_g2s(wring + static_cast<size_t>(pos + t) * p.blob_bytes,
                                     p.wp + static_cast<size_t>(e[t] >> 4) * 16, ((e[t + 1] >> 4) - (e[t] >> 4)) * 16u,
                                     fbar, policy);
                } else if (kWeights) {
                    mbar_arrive_expect_tx(fbar, static_cast<uint32_t>(c * p.blob_bytes));
                    bulk_g2s(wring + static_cast<size_t>(pos) * p.blob_bytes,
                             wtile + static_cast<size_t>(kb) * p.blob_bytes, static_cast<uint32_t>(c * p.blob_bytes),
                             fbar, policy);
                } else {
                    mbar_arrive_expect_tx(fbar, static_cast<uint32_t>(c * p.act_slot));
                    tma_load_3d(aring + static_cast<size_t>(pos) * p.act_slot, &maps->m[c - 1], 0, mt * p.tile_m,
                                (MODE == kModeW4A8) ? kb : 2 * kb, fbar);
                }
                armed = ch + 1;
            }
            ++ch;
            cb.next();
            kb += c;
            pos += c;
            if (pos == p.slots) {
                pos = 0;
                if (first_pass_chunks == 0xffffffffu) first_pass_chunks = ch;
            }
        }
    }
    // wind-down: every copy this CTA started must land before the CTA exits (after an expired
    // wait, one more bounded wait is the most this spends)
    for (uint32_t k = armed > kChunkBars ? armed - kChunkBars : 0; k < armed; ++k)
        if (!wait_bar(&b.full[chunk_bar(k)], chunk_parity(k), ctl, false)) break;
}

template <int MODE>
__device__ void issuer_role(int q, const GemmArgs& p, const uint8_t* aring, Barriers& b, uint32_t tmem,
                            const Ctl& ctl, long long beg, long long end) {
    constexpr int kSteps = (MODE == kModeW4A8) ? 4 : 8;          // MMA K: 32 int8 or 16 fp16
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;
    const uint32_t idesc = (MODE == kModeW4A8) ? idesc_s8_s32(kTileN, p.tile_m) : idesc_f16_f32(kTileN, p.tile_m);
    const int steps = kSteps / p.issuers;
    const int k0 = q * steps;                                     // first k-step of this issuer
    const int hw = (p.issuers == 1) ? -1 : (k0 * (kSteps == 8 ? 16 : 32)) / 64;  // A half it needs (-1: both)
    const uint32_t d_tmem = tmem + static_cast<uint32_t>(q * p.tile_m);
    const uint32_t a_base = smem_addr(aring);
    ChunkBar cb;
    uint32_t iter = 0;
    int pos = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        bool first = true;
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, iter == 0);
            if (ok) ok = wait_bar(&b.full[cb.bar], cb.parity, ctl);
            cb.next();
            for (int t = 0; t < c; ++t, ++iter) {
                const int s = pos + t;
                const uint32_t a = iter % kASlots, aph = (iter / kASlots) & 1;
                if (ok) {
                    if (hw >= 0) {
                        ok = wait_bar(&b.afull[a][hw], aph, ctl);
                    } else {
                        ok = wait_bar(&b.afull[a][0], aph, ctl);
                        if (ok) ok = wait_bar(&b.afull[a][1], aph, ctl);
                    }
                }
                if (!ok) continue;
                tc_fence_after();
                const uint32_t act = a_base + static_cast<uint32_t>(s * p.act_slot);
                const uint32_t a_tmem = tmem + kTmemAOffset + a * kSlotCols;
                const uint64_t bdesc0 = smem_desc_sw128(act);
                for (int kk = k0; kk < k0 + steps; ++kk) {
                    const uint32_t boff = (MODE == kModeW4A8)
                                              ? static_cast<uint32_t>(kk * 32)
                                              : static_cast<uint32_t>((kk >> 2) * p.tile_m * 128 + (kk & 3) * 32);
                    const uint64_t bdesc = smem_desc_advance(bdesc0, boff);
                    const uint32_t accumulate = first ? 0u : 1u;
                    first = false;
                    if (MODE == kModeW4A8)
                        mma_i8_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, accumulate);
                    else
                        mma_f16_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, accumulate);
                }
                tc_commit(&b.aempty[a]);
                tc_commit(&b.empty_a[s]);
            }
            kb += c;
            pos += c;
            if (pos == p.slots) pos = 0;
        }
        if (ok) tc_commit(&b.dfull);
    }
    tc_commit(&b.drain[q]);
    wait_bar(&b.drain[q], 0, ctl, false);
}

// ------------------------------------------------------------------ kernels
__device__ __forceinline__ uint8_t* align_ring(uint8_t* smem_dyn) {
    const uint32_t raw = smem_addr(smem_dyn);
    return smem_dyn + ((1024u - (raw & 1023u)) & 1023u);  // swizzle atoms need 1024-byte alignment
}

// Number of weight blobs each CTA asks L2 to prefetch at kernel entry: HBM starts streaming
// the first k-blocks while the CTA initialises barriers and tensor memory, and, when the
// kernel was launched early behind another one of the stream, while that one finishes.
// (A prefetch only fills L2, the point of coherence: it cannot observe stale data.)
constexpr int kPrefetchBlobs = 24;

template <bool kMix = false>
__device__ void prefetch_first_blobs(const GemmArgs& p, long long beg, long long end) {
    if (kMix) {  // blobs of varying size: the CTA's table entries (16-byte aligned, inside the table)
        const long long lo = (beg * 4) & ~15ll, hi = ((end + 1) * 4 + 15) & ~15ll;
        if (hi > lo) prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(p.mix_table) + lo, static_cast<uint32_t>(hi - lo));
        return;
    }
    SegCursor seg(beg, end, p.k_blocks);
    int left = kPrefetchBlobs;
    while (left > 0 && seg.next()) {
        const int nt = seg.tile / p.m_tiles;
        int n = seg.kb_hi - seg.kb_lo + 1;
        if (n > left) n = left;
        prefetch_l2_bulk(p.wp + (static_cast<size_t>(nt) * p.k_blocks + seg.kb_lo) * p.blob_bytes,
                         static_cast<uint32_t>(n * p.blob_bytes));
        left -= n;
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsLarge, 1)
    wq_gemm_large(const __grid_constant__ ActMaps maps, const GemmArgs p) {
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Barriers bars;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    uint8_t* aring = align_ring(smem_dyn);
    uint8_t* wring = aring + static_cast<size_t>(p.slots) * p.act_slot;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const long long beg = unit_start(blockIdx.x, p.units, p.grid);
    const long long end = unit_start(blockIdx.x + 1, p.units, p.grid);
    if (threadIdx.x == 0) griddep_launch_dependents();
    if (warp == kWeightWarp && lane == 0) prefetch_first_blobs(p, beg, end);
    if (warp == 0) {  // the lanes of warp 0 initialise the barriers side by side
        for (int k = lane; k < kChunkBars; k += 32) mbar_init(&bars.full[k], 2);
        for (int s = lane; s < p.slots; s += 32) {
            mbar_init(&bars.empty_w[s], kNumDqWarps / kDqResidues);  // the k-block's dequant group
            mbar_init(&bars.empty_a[s], p.issuers);
        }
        if (lane < kASlots) {
            mbar_init(&bars.afull[lane][0], 4);
            mbar_init(&bars.afull[lane][1], 4);
            mbar_init(&bars.aempty[lane], p.issuers);
        }
        if (lane == 0) {
            mbar_init(&bars.dfull, p.issuers);
            abort_flag = 0;
        }
        if (lane < kMaxIssuers) mbar_init(&bars.drain[lane], 1);
        fence_barrier_init();
    }
    if (warp == kIssuerWarp0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kActWarp && lane == 0)
        for (int c = 0; c < p.chunk; ++c) prefetch_tensor_map(&maps.m[c]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const Ctl ctl{&abort_flag, p.status, p.timeout_ns};

    if (warp < kNumDqWarps) {
        dequant_role<MODE>(p, wring, bars, tmem, ctl, beg, end);
    } else if (warp < kIssuerWarp0 + kMaxIssuers) {
        const int q = warp - kIssuerWarp0;
        if (q < p.issuers && lane == 0) issuer_role<MODE>(q, p, aring, bars, tmem, ctl, beg, end);
    } else if (warp == kWeightWarp) {
        if (lane == 0) producer_role<MODE, true>(&maps, p, aring, wring, bars, ctl, beg, end);
    } else {
        if (lane == 0) producer_role<MODE, false>(&maps, p, aring, wring, bars, ctl, beg, end);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kIssuerWarp0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ small tiles
// Small tiles (at most 32 rows of A) split the walk's k-blocks round-robin over 4 residues: walk
// index i belongs to residue r = i mod 4. Residue r owns one dequantised A slot and two partial
// buffers (2r, 2r + 1) in tensor memory, one MMA issuer and one dequant warp per lane quarter;
// so every mbarrier has fixed participants that see all of its phases in order (a parity wait
// can never pass on a phase two ahead or behind).
//
// Per k-block i of residue r (the u-th of that residue, u = i / 4):
//   dequant warps (4 quarters): wait for the chunk's copies (full), read the 16 code words of
//     their column and release the ring slot (empty_w); wait until the MMAs of their previous
//     k-block are done (aempty[r], phase u - 1): that frees A slot r and completes partial
//     buffer 2r + (u - 1) % 2; dequantise k-block i into A slot r and signal afull[r]; then,
//     while the MMAs of k-block i run into the other buffer, add partial u - 1 into fp32
//     (int32) registers with that k-block's group scale.
//   issuer r: wait for the activations (full) and afull[r] (phase u), issue the 8 MMAs
//     (K = 16 each) of the k-block into partial buffer 2r + u % 2, commit aempty[r] and the
//     ring slot's activation half (empty_a).
// The next MMA into buffer 2r + (u - 1) % 2 is that of k-block u + 1, which waits for afull[r]
// phase u + 1: the dequant warps signal it only after they have read partial u - 1.
// At a segment's end each dequant warp waits for its last MMA and adds that partial too; the
// 4 residue warps of a quarter then sum their registers through tensor memory (fixed order
// r = 0..3) and each finishes a quarter of the tile rows in the epilogue.
__device__ __forceinline__ bool chunk_has(uint32_t iter0, int c, uint32_t period, uint32_t residue) {
    return ((residue + period - iter0 % period) % period) < static_cast<uint32_t>(c);
}

// Rows of the tile below M (tiles past the last full one are partly padding).
__device__ __forceinline__ int live_rows(const GemmArgs& p, int tile, int TM) {
    const int live = p.M - (tile % p.m_tiles) * TM;
    return live < TM ? live : TM;
}

// Adds the partial buffer at paddr (this warp's lane quarter) into acc, the first `live` columns only.
template <int MODE, int TM>
__device__ __forceinline__ void add_partial(uint32_t (&acc)[TM], uint32_t paddr, float sc, int live) {
#pragma unroll
    for (int c0 = 0; c0 < TM; c0 += 8) {
        if (c0 < live) {  // warp-uniform
            uint32_t v[8];
            tmem_ld_x8(paddr + static_cast<uint32_t>(c0), v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if (MODE == kModeW4A8)
                    acc[c0 + c] = static_cast<uint32_t>(static_cast<int32_t>(acc[c0 + c]) + static_cast<int32_t>(v[c]));
                else
                    acc[c0 + c] = __float_as_uint(fmaf(sc, __uint_as_float(v[c]), __uint_as_float(acc[c0 + c])));
            }
        }
    }
}

// Epilogue of a small tile for one residue warp: lane l of the warp in lane quarter q holds in
// v the complete sums of output column n = tile*128 + 32q + l for the tile rows r*TM/4 ..
// r*TM/4 + TM/4 - 1. Only rows below M are stored, published or fetched.
//
// A CTA that does not own the tile writes its partial rows to its workspace slot and (after
// all 16 dequant warps have written) releases its flag. The owner finds the contributing CTAs
// directly (those before it whose unit range reaches into the tile), lets each lane poll one
// contributor's flag, then adds the contributors' partials in descending CTA order with
// several contributors' loads in flight at a time.
template <int MODE, int TM>
__device__ void epilogue_small(const GemmArgs& p, const Ctl& ctl, const SegCursor& seg, uint32_t (&v)[TM / 4], bool ok,
                               int quarter, int lane, int r) {
    constexpr int H = TM / 4;
    constexpr int kBatch = (H <= 4) ? 4 : 2;  // contributors whose loads are in flight together
    const int row = quarter * 32 + lane;
    const int nt = seg.tile / p.m_tiles, mt = seg.tile % p.m_tiles;
    const int n = nt * kTileN + row;
    const int r0 = r * H;  // first tile row of this warp
    int live = live_rows(p, seg.tile, TM) - r0;
    live = live < 0 ? 0 : (live > H ? H : live);
    const bool leader = threadIdx.x == 0;
    const int me = static_cast<int>(blockIdx.x);
    if (!seg.owner) {
        uint32_t* part = reinterpret_cast<uint32_t*>(p.ws_partial) + static_cast<size_t>(me) * TM * kTileN;
        if (ok) {
#pragma unroll
            for (int c = 0; c < H; ++c)
                if (c < live) part[static_cast<size_t>(r0 + c) * kTileN + row] = v[c];
        }
        // the barrier orders every thread's partial stores before the leader's (cumulative) release
        named_barrier_sync(2, kDqWarpsS * 32);
        if (leader && ok && !*ctl.abort_flag && me != p.skip_publish) st_release_gpu(&p.ws_flags[me], 1);
        return;
    }
    int c_last = me;  // contributors are CTAs c_last .. me - 1
    if (!seg.whole) {
        // the CTA holding the tile's first unit: the smallest c with unit_start(c + 1) > tbase
        const long long tbase = static_cast<long long>(seg.tile) * p.k_blocks;
        c_last = static_cast<int>(((tbase + 1) * p.grid + p.units - 1) / p.units) - 1;
        const int ncontrib = me - c_last;
        for (int j0 = 0; j0 < ncontrib; j0 += 32) {
            bool good = true;
            if (ok && j0 + lane < ncontrib) good = wait_flag(&p.ws_flags[me - 1 - j0 - lane], ctl);
            ok = __all_sync(0xffffffffu, good) && ok;
        }
        __syncwarp();  // the polling lanes' acquires order the whole warp's loads below
        if (ok && live > 0) {
            for (int j = 0; j < ncontrib; j += kBatch) {
                uint32_t w[kBatch][H];
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const uint32_t* part = reinterpret_cast<const uint32_t*>(p.ws_partial) +
                                           static_cast<size_t>(me - 1 - j - b) * TM * kTileN;
#pragma unroll
                    for (int c = 0; c < H; ++c)
                        w[b][c] = (j + b < ncontrib && c < live)
                                      ? __ldcg(part + static_cast<size_t>(r0 + c) * kTileN + row)
                                      : 0u;
                }
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    if (j + b < ncontrib) {
#pragma unroll
                        for (int c = 0; c < H; ++c) {
                            if (MODE == kModeW4A8)
                                v[c] = static_cast<uint32_t>(static_cast<int32_t>(v[c]) + static_cast<int32_t>(w[b][c]));
                            else
                                v[c] = __float_as_uint(__uint_as_float(v[c]) + __uint_as_float(w[b][c]));
                        }
                    }
                }
            }
        }
    }
    if (ok && n < p.N) {
        float s_col = 1.0f, sw_col = 0.0f;
        if (MODE == kModeChannel) s_col = __half2float(__ushort_as_half(p.s_chan[n]));
        if (MODE == kModeW4A8) sw_col = p.sw[n];
#pragma unroll
        for (int c = 0; c < H; ++c) {
            if (c < live) {
                const int m = mt * TM + r0 + c;
                const size_t o = static_cast<size_t>(m) * p.N + n;
                float y;
                if (MODE == kModeW4A8) {
                    const int32_t a = static_cast<int32_t>(v[c]) >> 4;
                    if (p.acc_out) p.acc_out[o] = a;
                    const float t = static_cast<float>(a) * p.sa[m];
                    y = t * sw_col;
                } else if (MODE == kModeChannel) {
                    y = __uint_as_float(v[c]) * s_col;
                } else {
                    y = __uint_as_float(v[c]);
                }
                p.y[o] = __half_as_ushort(__float2half_rn(y));
            }
        }
    }
    if (!seg.whole) {
        named_barrier_sync(2, kDqWarpsS * 32);  // every dequant warp has read the partials
        if (leader && !*ctl.abort_flag)  // as in the large-tile epilogue: not after an expired wait
            for (int cc = me - 1; cc >= c_last; --cc) p.ws_flags[cc] = 0;
    }
}

// Dequant (and accumulate) warp of a small tile: lane quarter = warp % 4, residue r = warp / 4.
// kScaled: the group scale multiplies the fp16 weight (g < 128); otherwise group scales
// (g >= 128) multiply each k-block's fp32 partial as it is added.
template <int MODE, int TM, bool kScaled>
__device__ void dequant_role_small(const GemmArgs& p, const uint8_t* wring, Barriers& b, uint32_t tmem,
                                   const Ctl& ctl, long long beg, long long end) {
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;  // 128 k of fp16 or int8 per lane
    constexpr int H = TM / 4;
    constexpr bool kScaleAtAdd = is_group(MODE) && !kScaled;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    const uint32_t r = static_cast<uint32_t>(warp >> 2);
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t slot_addr = tmem + lane_base + kTmemAOffsetS + r * kSlotCols;  // A slot r, this quarter
    const uint32_t part_base = tmem + lane_base + 2 * r * TM;  // partial buffers 2r, 2r + 1 (by use parity)
    ChunkBar cb;
    uint32_t iter = 0, uses = 0;  // uses: k-blocks of residue r handed to the MMA so far
    int pos = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        const int live = live_rows(p, seg.tile, TM);
        uint32_t acc[TM];
#pragma unroll
        for (int c = 0; c < TM; ++c) acc[c] = 0;  // +0.0f and int 0 share the bit pattern
        bool pending = false;                      // a k-block of this segment whose partial is not added yet
        float sc_pending = 1.0f;
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, iter == 0);
            const uint32_t fb = cb.bar, fpar = cb.parity;
            cb.next();
            if (chunk_has(iter, c, 4, r)) {
                if (ok) ok = __all_sync(0xffffffffu, wait_bar(&b.full[fb], fpar, ctl));
                const int t = static_cast<int>((r + 4 - iter % 4) % 4);  // this residue's k-block in the chunk
                const int s = pos + t;
                // TM = 32 keeps 32 accumulators live: it reads the code words one half at a time
                // (and so holds the ring slot until the second half is read)
                constexpr bool kSplitLoad = TM > 16;
                const uint8_t* blob = wring + static_cast<size_t>(s) * p.blob_bytes;
                const uint4* words = reinterpret_cast<const uint4*>(blob);
                const uint16_t* scs = reinterpret_cast<const uint16_t*>(blob + kCodeBytes);
                uint4 w[4];
                uint16_t sc[4] = {0, 0, 0, 0};
                uint16_t sc_add = 0;
                uint8_t zq[MODE == kModeGroupZP ? 4 : 1] = {8};  // asymmetric groups: each 32-row block's zero
                if (ok) {
#pragma unroll
                    for (int hv = 0; hv < (kSplitLoad ? 2 : 4); ++hv) w[hv] = words[hv * kTileN + row];
                    if (kScaled) {
#pragma unroll
                        for (int hv = 0; hv < 4; ++hv) sc[hv] = scs[((32 * hv) / p.group_rows) * kTileN + row];
                    }
                    if (kScaleAtAdd) sc_add = scs[row];
                    if constexpr (MODE == kModeGroupZP) {
                        if (kScaled) {
#pragma unroll
                            for (int hv = 0; hv < 4; ++hv)
                                zq[hv] = blob[p.zp_offset + ((32 * hv) / p.group_rows) * kTileN + row];
                        } else {
                            zq[0] = zq[1] = zq[2] = zq[3] = blob[p.zp_offset + row];
                        }
                    }
                }
                if (!kSplitLoad) {
                    __syncwarp();
                    if (ok && lane == 0) mbar_arrive(&b.empty_w[s]);
                }
                // MMAs of this residue's previous k-block done: A slot r is free, its partial complete
                if (ok) ok = __all_sync(0xffffffffu, wait_bar(&b.aempty[r], (uses & 1u) ^ 1u, ctl));
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (kSplitLoad && h == 1) {
                            w[0] = words[2 * kTileN + row];
                            w[1] = words[3 * kTileN + row];
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&b.empty_w[s]);
                        }
                        const int i0 = kSplitLoad ? 0 : 2 * h;
                        const uint32_t wv[8] = {w[i0].x,     w[i0].y,     w[i0].z,     w[i0].w,
                                                w[i0 + 1].x, w[i0 + 1].y, w[i0 + 1].z, w[i0 + 1].w};
                        if (MODE == kModeW4A8) {
                            uint32_t out[16];
#pragma unroll
                            for (int k = 0; k < 8; ++k) dequant_word_i8(wv[k], out + 2 * k);
                            tmem_st_x16(slot_addr + h * 16, out);
                        } else {
                            const __half2 s0 = __half2half2(__ushort_as_half(sc[2 * h]));
                            const __half2 s1 = __half2half2(__ushort_as_half(sc[2 * h + 1]));
#pragma unroll
                            for (int q2 = 0; q2 < 2; ++q2) {  // 16 registers per store keeps the live set small
                                uint32_t out[16];
                                if constexpr (MODE == kModeGroupZP) {
                                    const uint32_t zz = zq[2 * h + q2];
                                    const uint32_t klo = zp_lo(zz), khi = zp_hi(zz);
#pragma unroll
                                    for (int k = 0; k < 4; ++k)
                                        dequant_word_f16_zp(wv[4 * q2 + k], q2 == 0 ? s0 : s1, kScaled, klo, khi,
                                                            out + 4 * k);
                                } else {
#pragma unroll
                                    for (int k = 0; k < 4; ++k)
                                        dequant_word_f16(wv[4 * q2 + k], q2 == 0 ? s0 : s1, kScaled, out + 4 * k);
                                }
                                tmem_st_x16(slot_addr + h * 32 + q2 * 16, out);
                            }
                        }
                    }
                    tmem_st_wait();
                    tc_fence_before();
                } else if (kSplitLoad) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&b.empty_w[s]);  // a failed wait still releases the slot
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&b.afull[r][0]);
                // the previous k-block's partial, in the other buffer, while the MMAs of this
                // one run; the next MMA into that buffer waits for this warp's next afull
                if (ok && pending) add_partial<MODE, TM>(acc, part_base + ((uses - 1) & 1u) * TM, sc_pending, live);
                ++uses;
                pending = true;
                sc_pending = kScaleAtAdd ? __half2float(__ushort_as_half(sc_add)) : 1.0f;
            }
            iter += c;
            kb += c;
            pos += c;
            if (pos == p.slots) pos = 0;
        }
        // the segment's last k-block of this residue: wait for its MMAs and add its partial
        if (pending) {
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(&b.aempty[r], (uses & 1u) ^ 1u, ctl));
            if (ok) {
                tc_fence_after();
                add_partial<MODE, TM>(acc, part_base + ((uses - 1) & 1u) * TM, sc_pending, live);
            }
        }
        // the 4 residue warps of this quarter sum their registers (r = 0..3 in order) through
        // partial buffers 0, 2, 4, 6, each finishing TM/4 rows: buffer 2r holds no MMA result
        // now, and none is issued into it before this warp signals its next afull
        ok = ok && !*ctl.abort_flag;
        if constexpr (TM == 16)
            tmem_st_x16(part_base, acc);
        else
            tmem_st_x32(part_base, acc);
        tmem_st_wait();
        tc_fence_before();
        named_barrier_sync(3 + quarter, 4 * 32);
        tc_fence_after();
        uint32_t v[H];
#pragma unroll
        for (int c = 0; c < H; ++c) v[c] = 0;
        if (static_cast<int>(r) * H < live) {
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                uint32_t x[H];
                if constexpr (H == 4)
                    tmem_ld_x4(tmem + lane_base + 2 * rr * TM + r * H, x);
                else
                    tmem_ld_x8(tmem + lane_base + 2 * rr * TM + r * H, x);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < H; ++c)
                    v[c] = (MODE == kModeW4A8)
                               ? static_cast<uint32_t>(static_cast<int32_t>(v[c]) + static_cast<int32_t>(x[c]))
                               : __float_as_uint(__uint_as_float(v[c]) + __uint_as_float(x[c]));
            }
        }
        tc_fence_before();
        named_barrier_sync(3 + quarter, 4 * 32);  // all reads done before any MMA refills a buffer
        epilogue_small<MODE, TM>(p, ctl, seg, v, ok, quarter, lane, static_cast<int>(r));
    }
}

// Issuer r of a small tile: every k-block whose walk index is r mod 4 is its own; it waits for
// the k-block's activations (full) and its dequantised weights (A slot r), then writes the
// k-block's product into partial buffer 2r + (its use count mod 2) with a fresh accumulation.
template <int MODE, int TM>
__device__ void issuer_role_small(int r, const GemmArgs& p, const uint8_t* aring, Barriers& b, uint32_t tmem,
                                  const Ctl& ctl, long long beg, long long end) {
    constexpr int kSteps = (MODE == kModeW4A8) ? 4 : 8;
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;
    const uint32_t idesc = (MODE == kModeW4A8) ? idesc_s8_s32(kTileN, TM) : idesc_f16_f32(kTileN, TM);
    const uint32_t a_tmem = tmem + kTmemAOffsetS + static_cast<uint32_t>(r * kSlotCols);
    const uint32_t a_base = smem_addr(aring);
    ChunkBar cb;
    uint32_t iter = 0, uses = 0;
    int pos = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, iter == 0);
            const uint32_t fb = cb.bar, fpar = cb.parity;
            cb.next();
            if (chunk_has(iter, c, 4, static_cast<uint32_t>(r))) {
                const int t = static_cast<int>((static_cast<uint32_t>(r) + 4 - iter % 4) % 4);
                const int s = pos + t;
                if (ok) ok = wait_bar(&b.full[fb], fpar, ctl);
                if (ok) ok = wait_bar(&b.afull[r][0], uses & 1u, ctl);
                const uint32_t d_tmem = tmem + static_cast<uint32_t>((2 * r + static_cast<int>(uses & 1u)) * TM);
                ++uses;
                if (ok) {
                    tc_fence_after();
                    const uint32_t act = a_base + static_cast<uint32_t>(s * p.act_slot);
                    const uint64_t bdesc0 = smem_desc_sw128(act);
#pragma unroll
                    for (int kk = 0; kk < kSteps; ++kk) {
                        const uint32_t boff = (MODE == kModeW4A8)
                                                  ? static_cast<uint32_t>(kk * 32)
                                                  : static_cast<uint32_t>((kk >> 2) * TM * 128 + (kk & 3) * 32);
                        const uint64_t bdesc = smem_desc_advance(bdesc0, boff);
                        if (MODE == kModeW4A8)
                            mma_i8_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, kk != 0);
                        else
                            mma_f16_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, kk != 0);
                    }
                    tc_commit(&b.aempty[r]);
                    tc_commit(&b.empty_a[s]);
                }
            }
            iter += c;
            kb += c;
            pos += c;
            if (pos == p.slots) pos = 0;
        }
    }
    tc_commit(&b.drain[r]);
    wait_bar(&b.drain[r], 0, ctl, false);
}

// The small-tile protocol relies on one period (4) for dequant residues, A slots, issuers and
// partial buffers, and on the A slots fitting in tensor memory beside the partial buffers.
static_assert(kDqWarpsS == 16 && kASlotsS == kMaxIssuers && kMaxIssuers == 4, "small-tile periods");
static_assert(2 * kMaxIssuers * kSmallTileMax <= kTmemAOffsetS && kTmemAOffsetS + kASlotsS * 64 <= kTmemCols,
              "small-tile tensor-memory columns");
static_assert(kChunkBars > kMaxSlots && kMaxChunk <= 4, "one k-block per residue per chunk");

template <int MODE, int TM>
__global__ void __launch_bounds__(kThreadsSmall, 1)
    wq_gemm_small(const __grid_constant__ ActMaps maps, const GemmArgs p) {
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Barriers bars;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    uint8_t* aring = align_ring(smem_dyn);
    uint8_t* wring = aring + static_cast<size_t>(p.slots) * p.act_slot;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const long long beg = unit_start(blockIdx.x, p.units, p.grid);
    const long long end = unit_start(blockIdx.x + 1, p.units, p.grid);
    if (threadIdx.x == 0) griddep_launch_dependents();
    if (warp == kWeightWarpS && lane == 0) prefetch_first_blobs(p, beg, end);
    if (warp == 0) {  // the lanes of warp 0 initialise the barriers side by side
        for (int k = lane; k < kChunkBars; k += 32) mbar_init(&bars.full[k], 2);
        for (int s = lane; s < p.slots; s += 32) {
            mbar_init(&bars.empty_w[s], 4);  // the k-block's 4 dequant warps (one per lane quarter)
            mbar_init(&bars.empty_a[s], 1);  // the k-block's issuer
        }
        if (lane < kASlotsS) {
            mbar_init(&bars.afull[lane][0], 4);
            mbar_init(&bars.aempty[lane], 1);
            mbar_init(&bars.drain[lane], 1);
        }
        if (lane == 0) abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kIssuerWarp0S) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kActWarpS && lane == 0)
        for (int c = 0; c < p.chunk; ++c) prefetch_tensor_map(&maps.m[c]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const Ctl ctl{&abort_flag, p.status, p.timeout_ns};

    if (warp < kDqWarpsS) {
        if constexpr (is_group(MODE)) {
            if (p.scale_in_dequant)
                dequant_role_small<MODE, TM, true>(p, wring, bars, tmem, ctl, beg, end);
            else
                dequant_role_small<MODE, TM, false>(p, wring, bars, tmem, ctl, beg, end);
        } else {
            dequant_role_small<MODE, TM, false>(p, wring, bars, tmem, ctl, beg, end);
        }
    } else if (warp < kIssuerWarp0S + kMaxIssuers) {
        if (lane == 0) issuer_role_small<MODE, TM>(warp - kIssuerWarp0S, p, aring, bars, tmem, ctl, beg, end);
    } else if (warp == kWeightWarpS) {
        if (lane == 0) producer_role<MODE, true>(&maps, p, aring, wring, bars, ctl, beg, end);
    } else if (warp == kActWarpS) {
        if (lane == 0) producer_role<MODE, false>(&maps, p, aring, wring, bars, ctl, beg, end);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kIssuerWarp0S) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ register-operand tiles
// At M <= 8 a k-block's product is 128 x 128 x M multiply-adds: too little to amortise the
// tensor-memory chain of the small-tile kernel (dequantise into tensor memory, hand the slot
// to an issuing thread, wait for its MMAs, read the partial back), whose per-k-block cost, not
// HBM, bounds that kernel at small M. Here every warp multiplies the weights it has just
// dequantised, from its own registers, with the warp-level tensor-core instruction
// (mma.sync m16n8k16, fp16 operands, fp32 accumulation): no cross-warp chain, no tensor memory.
//
// Roles (576 threads): warps 0..15 consume every k-block of the walk. Warp w owns 16 weight
// columns 16 (w mod 8) + {0..7, 8..15} and the 64 rows 64 (w / 8) .. + 63 of each k-block (two
// 32-row blocks A and B); warp 16 streams the weight blobs and warp 17 the activation rows
// (unswizzled, TM rows of 128 k per k-block) into the shared-memory ring of the other kernels.
// Lane (g, q) = (lane / 4, lane % 4) loads word q of its two columns g, g + 8 in blocks A and
// B: four 32-bit loads, 8 rows each. Each word becomes four fp16 pairs of exact (q - z) (the
// magic-number conversion); pair s of the four words is exactly the lane's A fragment of the
// s-th MMA (rows = columns g, g + 8; k = the pair's two rows, block A in k 0..7, block B in
// k 8..15), and pair s of the lane's activation words (rows 8q .. 8q + 7 of blocks A and B of
// activation row g) its B fragment. The MMA's k order is a permutation of the 64 rows, the
// same for both operands. The four MMAs of a k-block accumulate in fp32; the group scale
// multiplies the k-block's sum (acc += s * D) for g >= 64, or the fp16 weight (g = 32, one
// rounding per weight as in the other kernels); per-column scales wait for the epilogue.
// At a segment's end the two row halves of each column are summed through shared memory (two
// buffers by segment parity) and warps 0..3 run the stream-K epilogue of the small tiles.

__device__ __forceinline__ void mma_m16n8k16_f16_f32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_m16n8k32_s8_s32(uint32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Epilogue of a register-operand tile: thread (quarter, lane) of warps 0..3 holds in v the
// complete sums of output column n = tile*128 + 32 quarter + lane for rows 0 .. TM - 1 (only
// rows below M are live). The stream-K protocol is that of the small tiles: a contributor
// writes its partial and releases its flag; the owner waits for its contributors' flags and
// adds their partials in descending CTA order.
template <int MODE, int TM>
__device__ void epilogue_rf(const GemmArgs& p, const Ctl& ctl, const SegCursor& seg, uint32_t (&v)[TM], bool ok,
                            int quarter, int lane) {
    const int row = quarter * 32 + lane;
    const int n = seg.tile * kTileN + row;  // one m-tile: tile index = n-tile index
    const int live = p.M < TM ? p.M : TM;
    const bool leader = threadIdx.x == 0;
    const int me = static_cast<int>(blockIdx.x);
    if (!seg.owner) {
        uint32_t* part = reinterpret_cast<uint32_t*>(p.ws_partial) + static_cast<size_t>(me) * TM * kTileN;
        if (ok) {
#pragma unroll
            for (int m = 0; m < TM; ++m)
                if (m < live) part[m * kTileN + row] = v[m];
        }
        // the barrier orders every thread's partial stores before the leader's (cumulative) release
        named_barrier_sync(2, 4 * 32);
        if (leader && ok && !*ctl.abort_flag && me != p.skip_publish) st_release_gpu(&p.ws_flags[me], 1);
        return;
    }
    int c_last = me;  // contributors are CTAs c_last .. me - 1
    if (!seg.whole) {
        const long long tbase = static_cast<long long>(seg.tile) * p.k_blocks;
        c_last = static_cast<int>(((tbase + 1) * p.grid + p.units - 1) / p.units) - 1;
        const int ncontrib = me - c_last;
        for (int j0 = 0; j0 < ncontrib; j0 += 32) {
            bool good = true;
            if (ok && j0 + lane < ncontrib) good = wait_flag(&p.ws_flags[me - 1 - j0 - lane], ctl);
            ok = __all_sync(0xffffffffu, good) && ok;
        }
        __syncwarp();  // the polling lanes' acquires order the whole warp's loads below
        if (ok) {
            constexpr int kBatch = TM <= 2 ? 4 : 2;
            for (int j = 0; j < ncontrib; j += kBatch) {
                uint32_t w[kBatch][TM];
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const uint32_t* part =
                        reinterpret_cast<const uint32_t*>(p.ws_partial) + static_cast<size_t>(me - 1 - j - b) * TM * kTileN;
#pragma unroll
                    for (int m = 0; m < TM; ++m) w[b][m] = (j + b < ncontrib && m < live) ? __ldcg(part + m * kTileN + row) : 0u;
                }
#pragma unroll
                for (int b = 0; b < kBatch; ++b)
                    if (j + b < ncontrib) {
#pragma unroll
                        for (int m = 0; m < TM; ++m)
                            v[m] = (MODE == kModeW4A8)
                                       ? static_cast<uint32_t>(static_cast<int32_t>(v[m]) + static_cast<int32_t>(w[b][m]))
                                       : __float_as_uint(__uint_as_float(v[m]) + __uint_as_float(w[b][m]));
                    }
            }
        }
    }
    if (ok && n < p.N) {
        const float s_col = (MODE == kModeChannel) ? __half2float(__ushort_as_half(p.s_chan[n])) : 1.0f;
        const float sw_col = (MODE == kModeW4A8) ? p.sw[n] : 0.0f;
#pragma unroll
        for (int m = 0; m < TM; ++m)
            if (m < live) {
                const size_t o = static_cast<size_t>(m) * p.N + n;
                float y;
                if (MODE == kModeW4A8) {
                    const int32_t acc = static_cast<int32_t>(v[m]) >> 4;  // the codes were 16 (q - 8)
                    if (p.acc_out) p.acc_out[o] = acc;
                    y = (static_cast<float>(acc) * p.sa[m]) * sw_col;
                } else {
                    y = (MODE == kModeChannel) ? __uint_as_float(v[m]) * s_col : __uint_as_float(v[m]);
                }
                p.y[o] = __half_as_ushort(__float2half_rn(y));
            }
    }
    if (!seg.whole) {
        named_barrier_sync(2, 4 * 32);  // every epilogue warp has read the partials
        if (leader && !*ctl.abort_flag)
            for (int cc = me - 1; cc >= c_last; --cc) p.ws_flags[cc] = 0;
    }
}

// How the register-operand consumer applies the group scale.
enum RfScale : int {
    kRfScaleNone = 0,     // per-column scales: the epilogue multiplies
    kRfScaleWeight = 1,   // g = 32: the fp16 weight (one rounding per weight)
    kRfScalePair = 2,     // g = 64: each 64-row pair's fp32 sum
    kRfScaleBlock = 3,    // g >= 128: each k-block's fp32 sum
};

// Pair s (rows 2s, 2s + 1 of the word's 8) of a code word as fp16 (q - z), with the constants
// klo = zp_lo(z), khi = zp_hi(z) and x8 = x >> 8; times the fp16 scale sc when kScaled. The
// four pairs of a word are dequant_word_f16_zp's four outputs, one at a time, so that the
// register-operand consumer builds each MMA's A fragment from the same pair of four words.
template <int S, bool kScaled>
__device__ __forceinline__ uint32_t pair_f16(uint32_t x, uint32_t x8, uint32_t klo, uint32_t khi, __half2 sc) {
    const uint32_t kMagic = 0x64006400u;
    const __half2 kSixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    __half2 h;
    if constexpr (S == 0) {
        const uint32_t u = lop3_and_or(x, 0x000F000Fu, kMagic);
        h = __hsub2(half2_bits(u), half2_bits(klo));
    } else if constexpr (S == 1) {
        const uint32_t u = lop3_and_or(x, 0x00F000F0u, kMagic);
        h = __hfma2(half2_bits(u), kSixteenth, half2_bits(khi));
    } else if constexpr (S == 2) {
        const uint32_t u = lop3_and_or(x8, 0x000F000Fu, kMagic);
        h = __hsub2(half2_bits(u), half2_bits(klo));
    } else {
        const uint32_t u = lop3_and_or(x8, 0x00F000F0u, kMagic);
        h = __hfma2(half2_bits(u), kSixteenth, half2_bits(khi));
    }
    if constexpr (kScaled) h = __hmul2(h, sc);
    return *reinterpret_cast<uint32_t*>(&h);
}

// The two MMAs (t = 0, 1) of one row tile (columns c, c + 8 of lane (g, q): word x0 of column c,
// x1 of column c + 8, rows 8q .. 8q + 7 of a 32-row block) and one block. MMA t takes rows
// 8q + 4t .. 8q + 4t + 3 of each lane: its A fragment is pairs 2t and 2t + 1 of the two words
// (fragment k 2q, 2q + 1 and 2q + 8, 2q + 9), its B fragment pairs 2t and 2t + 1 of the lane's
// activation word of the same rows, two adjacent registers of one 16-byte load. The MMA's k order
// is a permutation of the block's rows, the same for both operands.
template <bool kScaled, int NB>
__device__ __forceinline__ void rf_mma_block(uint32_t x0, uint32_t x1, uint32_t klo0, uint32_t khi0, uint32_t klo1,
                                             uint32_t khi1, __half2 sc0, __half2 sc1, const uint4 (&act)[NB],
                                             float (&d)[NB][4]) {
    const uint32_t x80 = x0 >> 8, x81 = x1 >> 8;
    {
        const uint32_t afrag[4] = {pair_f16<0, kScaled>(x0, x80, klo0, khi0, sc0), pair_f16<0, kScaled>(x1, x81, klo1, khi1, sc1),
                                   pair_f16<1, kScaled>(x0, x80, klo0, khi0, sc0), pair_f16<1, kScaled>(x1, x81, klo1, khi1, sc1)};
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_m16n8k16_f16_f32(d[nb], afrag, act[nb].x, act[nb].y);
    }
    {
        const uint32_t afrag[4] = {pair_f16<2, kScaled>(x0, x80, klo0, khi0, sc0), pair_f16<2, kScaled>(x1, x81, klo1, khi1, sc1),
                                   pair_f16<3, kScaled>(x0, x80, klo0, khi0, sc0), pair_f16<3, kScaled>(x1, x81, klo1, khi1, sc1)};
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_m16n8k16_f16_f32(d[nb], afrag, act[nb].z, act[nb].w);
    }
}

// W4A8: the MMA (k = 32) of one row tile and one 32-row block. dequant_word_i8 gives a word's
// rows 8q .. 8q + 3 and 8q + 4 .. 8q + 7 as int8 16 (q - 8) in two registers: fragment k 4q .. 4q + 3
// and 4q + 16 .. 4q + 19; the activation word (8 int8 of the same rows) is the B fragment.
template <int NB>
__device__ __forceinline__ void rf_mma_block_i8(uint32_t x0, uint32_t x1, const uint2 (&act)[NB], uint32_t (&d)[NB][4]) {
    uint32_t o0[2], o1[2];
    dequant_word_i8(x0, o0);
    dequant_word_i8(x1, o1);
    const uint32_t afrag[4] = {o0[0], o1[0], o0[1], o1[1]};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) mma_m16n8k32_s8_s32(d[nb], afrag, act[nb].x, act[nb].y);
}

// 2:4 sparse weights. The sparse warp MMA (m16n8k32, groups of 4 along k, 2 kept per group)
// takes as A operand the kept values only: lane (g, q) holds, as four fp16 pairs, the two kept
// values of group q of rows g and g + 8, then of group q + 4 of the same rows, which is the
// order of the nibble pairs (0, 4), (1, 5), (2, 6), (3, 7) of one sparse code word: the word
// dequantises straight into the operand. Its metadata (lanes q = 0, 1 of each quad, selector 0)
// gives each group's two kept positions. The B operand is the dense 32 x 8 activation block:
// lane (g, q) register r holds activation row g, k = 8r + 2q, 8r + 2q + 1, i.e. element
// (g, 2q) of the 8 x 8 matrix at k = 8r: one ldmatrix.x4 per 8 activation rows.
__device__ __forceinline__ void mma_sp_m16n8k32_f16_f32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[4],
                                                        uint32_t e) {
    asm volatile(
        "mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9, %10, %11}, {%0, %1, %2, %3}, %12, 0x0;\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&d)[4], uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(saddr)
                 : "memory");
}

// The sparse MMA of one row tile (sparse code word x, metadata e) and one 32-row block; sc0,
// sc1: the fp16 scales of the tile's columns g and g + 8 when kScaled.
template <bool kScaled, int NB>
__device__ __forceinline__ void rf_sp_mma_block(uint32_t x, uint32_t e, __half2 sc0, __half2 sc1,
                                                const uint32_t (&bf)[NB][4], float (&d)[NB][4]) {
    const uint32_t x8 = x >> 8, klo = zp_lo(8), khi = zp_hi(8);
    const uint32_t a[4] = {pair_f16<0, kScaled>(x, x8, klo, khi, sc0), pair_f16<1, kScaled>(x, x8, klo, khi, sc1),
                           pair_f16<2, kScaled>(x, x8, klo, khi, sc0), pair_f16<3, kScaled>(x, x8, klo, khi, sc1)};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) mma_sp_m16n8k32_f16_f32(d[nb], a, bf[nb], e);
}

// Mixed 2/4-bit weights, a 2-bit block: lane (g, q) holds in one word the 2-bit codes of rows
// 8q .. 8q + 7 of columns g and g + 8 of its row tile, the fp16 pair (rows 8q + 2s, + 1) of
// column g in fields (s, s + 8) and of column g + 8 in fields (s + 4, s + 12). Field pair P
// (0..3) of a word y (the word, or the word shifted right by 8 for column g + 8): masking
// (3 << 2P) in each 16-bit half and OR-ing 0x6400 gives 1024 + 4^P q exactly, and
// u * 4^-P - (1024 / 4^P + 2) is q - 2 exactly (one fused multiply-add).
template <int P, bool kScaled>
__device__ __forceinline__ uint32_t pair2_f16(uint32_t y, __half2 sc) {
    const uint32_t u = lop3_and_or(y, (0x3u << (2 * P)) * 0x10001u, 0x64006400u);
    __half2 h;
    if constexpr (P == 0) {
        h = __hsub2(half2_bits(u), half2_bits(0x64026402u));  // - 1026
    } else {
        constexpr uint32_t kMul = P == 1 ? 0x34003400u : (P == 2 ? 0x2C002C00u : 0x24002400u);  // 1/4, 1/16, 1/64
        constexpr uint32_t kAdd = P == 1 ? 0xDC08DC08u : (P == 2 ? 0xD420D420u : 0xCC80CC80u);  // -258, -66, -18
        h = __hfma2(half2_bits(u), half2_bits(kMul), half2_bits(kAdd));
    }
    if constexpr (kScaled) h = __hmul2(h, sc);
    return *reinterpret_cast<uint32_t*>(&h);
}

// The two MMAs of one row tile and one 32-row 2-bit block: MMA t takes pairs 2t, 2t + 1 of both
// columns, the same k order as the 4-bit path, so the B fragments are the same registers.
template <bool kScaled, int NB>
__device__ __forceinline__ void rf_mma_block_2b(uint32_t x, __half2 sc0, __half2 sc1, const uint4 (&act)[NB],
                                                float (&d)[NB][4]) {
    const uint32_t x8 = x >> 8;
    {
        const uint32_t afrag[4] = {pair2_f16<0, kScaled>(x, sc0), pair2_f16<0, kScaled>(x8, sc1),
                                   pair2_f16<1, kScaled>(x, sc0), pair2_f16<1, kScaled>(x8, sc1)};
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_m16n8k16_f16_f32(d[nb], afrag, act[nb].x, act[nb].y);
    }
    {
        const uint32_t afrag[4] = {pair2_f16<2, kScaled>(x, sc0), pair2_f16<2, kScaled>(x8, sc1),
                                   pair2_f16<3, kScaled>(x, sc0), pair2_f16<3, kScaled>(x8, sc1)};
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_m16n8k16_f16_f32(d[nb], afrag, act[nb].z, act[nb].w);
    }
}

// Formats of the register-operand kernel's weights.
enum RfFmt : int { kFmtDense = 0, kFmtSparse = 1, kFmtMixed = 2 };

// Consumer warp of a register-operand tile (warps 0..15): residue r = warp / 4 takes the walk's
// k-blocks i with i mod 4 = r; column group cg = warp mod 4 owns columns 32 cg .. 32 cg + 31
// of every such k-block, all 128 rows. Lane (g, q) handles two MMA row tiles (columns
// 32 cg + 16 tau + g and + 8, tau = 0, 1) in each of the four 32-row blocks.
// red: 4 x TM x 128 floats of shared memory (residue, row, column).
// FMT kFmtSparse: 2:4 sparse blobs. Lane (g, q) then reads, per 32-row block and row tile, one
// code word and one metadata word, and the activation slot holds AR = max(TM, 8) rows in the
// 128-byte swizzled layout of the copy engine (16-byte chunk c of row m at chunk c ^ (m mod 8)),
// so that the eight rows of each 8 x 8 matrix of an ldmatrix fall in eight different banks.
// FMT kFmtMixed: mixed 2/4-bit blobs; the slot's widths word says which 32-row blocks are 4-bit
// (read as in a W4A16 blob) and which 2-bit (one word per row tile and lane).
template <int MODE, int TM, int SCALE, int FMT>
__device__ void rf_role(const GemmArgs& p, const uint8_t* aring, const uint8_t* wring, Barriers& b, float* red,
                        const Ctl& ctl, long long beg, long long end) {
    constexpr bool SP = FMT == kFmtSparse, MIX = FMT == kFmtMixed;
    constexpr int NB = (TM + 7) / 8;  // MMAs of 8 activation rows per k-step
    constexpr int AR = (SP && TM < kSpMinActRows) ? kSpMinActRows : TM;  // activation rows per slot piece
    constexpr bool kScaled = SCALE == kRfScaleWeight;
    constexpr bool kPerBlock = SCALE == kRfScaleWeight || SCALE == kRfScalePair || MODE == kModeGroupZP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t r = static_cast<uint32_t>(warp >> 2);
    const int cg = warp & 3;
    const int g = lane >> 2, q = lane & 3;
    const int colb = 32 * cg + g;  // columns colb + 16 tau + 8 j
    int aoff[NB];                  // activation row 8 nb + g (clamped to TM - 1), rows 8q .. 8q + 7 of block A of pair 0
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int arow = 8 * nb + g < TM ? 8 * nb + g : TM - 1;
        aoff[nb] = arow * 128 + 16 * q;
    }
    // SP: lane l gives the address of row l mod 8 of matrix l / 8 (k = 8 (l / 8) of the block):
    // activation row 8 nb + l mod 8, 16-byte chunk 4 (hv mod 2) + l / 8, swizzled
    const int lrow = lane & 7, lmat = lane >> 3;
    const uint32_t sw_off[2] = {static_cast<uint32_t>(((0 + lmat) ^ lrow) << 4), static_cast<uint32_t>(((4 + lmat) ^ lrow) << 4)};
    ChunkBar cb;
    uint32_t iter = 0;
    int pos = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        float acc[2][NB][4];  // [tau][nb]: columns colb + 16 tau + {0, 8} x rows 8 nb + 2q + {0, 1}
        uint32_t iacc[2][NB][4];  // W4A8: the same, exact int32
#pragma unroll
        for (int tau = 0; tau < 2; ++tau)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc[tau][nb][0] = acc[tau][nb][1] = acc[tau][nb][2] = acc[tau][nb][3] = 0.0f;
                iacc[tau][nb][0] = iacc[tau][nb][1] = iacc[tau][nb][2] = iacc[tau][nb][3] = 0u;
            }
        for (int kb = seg.kb_lo; kb <= seg.kb_hi;) {
            const int c = chunk_len(p.chunk, kb, seg.kb_hi, pos, p.slots, iter == 0);
            const uint32_t fb = cb.bar, fpar = cb.parity;
            const int s = pos + static_cast<int>((r + 4 - iter % 4) % 4);  // this residue's k-block, if any
            const bool mine = chunk_has(iter, c, 4, r);
            cb.next();
            iter += c;
            kb += c;
            pos += c;
            if (pos == p.slots) pos = 0;
            if (!mine) continue;
            ok = __all_sync(0xffffffffu, ok && wait_bar(&b.full[fb], fpar, ctl));
            if (!ok) continue;  // an expired wait: the CTA winds down (nothing more is read or released)
            const uint8_t* blob = wring + static_cast<size_t>(s) * p.blob_bytes;
            const uint32_t* words = reinterpret_cast<const uint32_t*>(blob);
            const uint32_t wb = MIX ? (b.wbits[s] & 0xFu) : 0xFu;  // mixed: bit v set = block v is 4-bit
            const uint16_t* scs = reinterpret_cast<const uint16_t*>(
                blob + (SP ? kSpHeadBytes : (MIX ? kMixBlock2 * (4 + __popc(wb)) : kCodeBytes)));
            const uint8_t* act = aring + static_cast<size_t>(s) * p.act_slot;
            uint32_t w[4][2][2];  // [block hv][tau][j]: word q of column colb + 16 tau + 8 j
                                  // SP: [hv][tau][0] code word, [hv][tau][1] metadata word of row tile 2 cg + tau
#pragma unroll
            for (int hv = 0; hv < 4; ++hv)
#pragma unroll
                for (int tau = 0; tau < 2; ++tau) {
                    if constexpr (SP) {
                        const int tile16 = hv * 8 + 2 * cg + tau;
                        w[hv][tau][0] = words[tile16 * 32 + lane];
                        w[hv][tau][1] = words[kSpCodeBytes / 4 + tile16 * 16 + 2 * g + (q & 1)];
                    } else if constexpr (MIX) {
                        const uint32_t* blk = words + (kMixBlock2 / 4) * (hv + __popc(wb & ((1u << hv) - 1u)));
                        if ((wb >> hv) & 1u) {
#pragma unroll
                            for (int j = 0; j < 2; ++j) w[hv][tau][j] = blk[(colb + 16 * tau + 8 * j) * 4 + q];
                        } else {
                            w[hv][tau][0] = blk[(2 * cg + tau) * 32 + lane];
                            w[hv][tau][1] = 0u;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j) w[hv][tau][j] = words[(hv * kTileN + colb + 16 * tau + 8 * j) * 4 + q];
                    }
                }
            if constexpr (MODE == kModeW4A8) {
                // int8 activation rows of 128 bytes: row arow, block hv, word q at arow*128 + 32 hv + 8q
#pragma unroll
                for (int hv = 0; hv < 4; ++hv) {
                    uint2 a8[NB];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
                        a8[nb] = *reinterpret_cast<const uint2*>(act + (aoff[nb] - 16 * q) + 32 * hv + 8 * q);
                    if (hv == 3) {  // the last reads of this ring slot are issued: release it
                        __syncwarp();
                        mbar_arrive_if(&b.empty_w[s], lane == 0);
                        mbar_arrive_if(&b.empty_a[s], lane == 0);
                    }
#pragma unroll
                    for (int tau = 0; tau < 2; ++tau) rf_mma_block_i8<NB>(w[hv][tau][0], w[hv][tau][1], a8, iacc[tau]);
                }
                continue;
            }
            float scb[2][2] = {{1.0f, 1.0f}, {1.0f, 1.0f}};  // kRfScaleBlock: [tau][j]
            if (SCALE == kRfScaleBlock) {
#pragma unroll
                for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                    for (int j = 0; j < 2; ++j) scb[tau][j] = __half2float(__ushort_as_half(scs[colb + 16 * tau + 8 * j]));
            }
            float part[2][NB][4];
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) part[tau][nb][0] = part[tau][nb][1] = part[tau][nb][2] = part[tau][nb][3] = 0.0f;
#pragma unroll
            for (int hv = 0; hv < 4; ++hv) {  // 32-row block hv
                __half2 sc[2][2];    // [tau][j]
                uint32_t klo[2][2], khi[2][2];
#pragma unroll
                for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        sc[tau][j] = __half2half2(__ushort_as_half(0x3C00));
                        klo[tau][j] = zp_lo(8);
                        khi[tau][j] = zp_hi(8);
                    }
                if (kPerBlock) {
                    const int u = (32 * hv) / p.group_rows;
#pragma unroll
                    for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int col = colb + 16 * tau + 8 * j;
                            if (SCALE == kRfScaleWeight || SCALE == kRfScalePair)
                                sc[tau][j] = __half2half2(__ushort_as_half(scs[u * kTileN + col]));
                            if (MODE == kModeGroupZP) {
                                const uint32_t zz = blob[p.zp_offset + u * kTileN + col];
                                klo[tau][j] = zp_lo(zz);
                                khi[tau][j] = zp_hi(zz);
                            }
                        }
                }
                uint4 a16[NB];      // activation row 8 nb + g, rows 8q .. 8q + 7 of block hv
                uint32_t bf[NB][4];  // SP: the B operands (activation rows 8 nb .. 8 nb + 7)
                if constexpr (SP) {
                    const uint32_t piece = smem_addr(act) + (hv >> 1) * AR * 128 + sw_off[hv & 1];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) ldmatrix_x4(bf[nb], piece + (8 * nb + lrow) * 128);
                } else {
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
                        a16[nb] = *reinterpret_cast<const uint4*>(act + (hv >> 1) * TM * 128 + aoff[nb] + (hv & 1) * 64);
                }
                if (hv == 3) {  // the last reads of this ring slot are issued: release it
                    __syncwarp();
                    mbar_arrive_if(&b.empty_w[s], lane == 0);
                    mbar_arrive_if(&b.empty_a[s], lane == 0);
                }
#pragma unroll
                for (int tau = 0; tau < 2; ++tau) {
                    float (&dst)[NB][4] = (SCALE == kRfScalePair || SCALE == kRfScaleBlock) ? part[tau] : acc[tau];
                    if constexpr (SP)
                        rf_sp_mma_block<kScaled, NB>(w[hv][tau][0], w[hv][tau][1], sc[tau][0], sc[tau][1], bf, dst);
                    else if (MIX && !((wb >> hv) & 1u))
                        rf_mma_block_2b<kScaled, NB>(w[hv][tau][0], sc[tau][0], sc[tau][1], a16, dst);
                    else
                        rf_mma_block<kScaled, NB>(w[hv][tau][0], w[hv][tau][1], klo[tau][0], khi[tau][0], klo[tau][1],
                                                  khi[tau][1], sc[tau][0], sc[tau][1], a16, dst);
                    if (SCALE == kRfScalePair && (hv & 1)) {  // the 64-row pair (blocks hv - 1, hv) shares a group
                        const float s0 = __low2float(sc[tau][0]), s1 = __low2float(sc[tau][1]);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            acc[tau][nb][0] = fmaf(s0, part[tau][nb][0], acc[tau][nb][0]);
                            acc[tau][nb][1] = fmaf(s0, part[tau][nb][1], acc[tau][nb][1]);
                            acc[tau][nb][2] = fmaf(s1, part[tau][nb][2], acc[tau][nb][2]);
                            acc[tau][nb][3] = fmaf(s1, part[tau][nb][3], acc[tau][nb][3]);
                            part[tau][nb][0] = part[tau][nb][1] = part[tau][nb][2] = part[tau][nb][3] = 0.0f;
                        }
                    }
                }
            }
            if (SCALE == kRfScaleBlock) {  // one group for the whole k-block
#pragma unroll
                for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        acc[tau][nb][0] = fmaf(scb[tau][0], part[tau][nb][0], acc[tau][nb][0]);
                        acc[tau][nb][1] = fmaf(scb[tau][0], part[tau][nb][1], acc[tau][nb][1]);
                        acc[tau][nb][2] = fmaf(scb[tau][1], part[tau][nb][2], acc[tau][nb][2]);
                        acc[tau][nb][3] = fmaf(scb[tau][1], part[tau][nb][3], acc[tau][nb][3]);
                    }
            }
        }
        // the residues' sums of each column, added in the order r = 0..3 by warps 0..3
#pragma unroll
        for (int tau = 0; tau < 2; ++tau)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int m = 8 * nb + 2 * q + jj;
                    if (m < TM) {
                        uint32_t* rw = reinterpret_cast<uint32_t*>(red);
                        rw[(r * TM + m) * kTileN + colb + 16 * tau] =
                            MODE == kModeW4A8 ? iacc[tau][nb][jj] : __float_as_uint(acc[tau][nb][jj]);
                        rw[(r * TM + m) * kTileN + colb + 16 * tau + 8] =
                            MODE == kModeW4A8 ? iacc[tau][nb][2 + jj] : __float_as_uint(acc[tau][nb][2 + jj]);
                    }
                }
        named_barrier_sync(1, kRfWarps * 32);
        uint32_t v[TM];
        if (warp < 4) {
            const int col = warp * 32 + lane;
            const uint32_t* rw = reinterpret_cast<const uint32_t*>(red);
#pragma unroll
            for (int m = 0; m < TM; ++m) {
                v[m] = rw[m * kTileN + col];
#pragma unroll
                for (int rr = 1; rr < 4; ++rr) {
                    const uint32_t x = rw[(rr * TM + m) * kTileN + col];
                    v[m] = (MODE == kModeW4A8) ? static_cast<uint32_t>(static_cast<int32_t>(v[m]) + static_cast<int32_t>(x))
                                               : __float_as_uint(__uint_as_float(v[m]) + __uint_as_float(x));
                }
            }
        }
        named_barrier_sync(1, kRfWarps * 32);  // the sums are read: the next segment may write them
        if (warp < 4) {
            ok = ok && !*ctl.abort_flag;
            epilogue_rf<MODE, TM>(p, ctl, seg, v, ok, warp, lane);
        }
    }
}

template <int MODE, int TM, int FMT = kFmtDense>
__global__ void __launch_bounds__(kThreadsRf, 1) wq_gemm_rf(const __grid_constant__ ActMaps maps, const GemmArgs p) {
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Barriers bars;
    __shared__ int abort_flag;

    uint8_t* aring = align_ring(smem_dyn);
    uint8_t* wring = aring + static_cast<size_t>(p.slots) * p.act_slot;
    float* red = reinterpret_cast<float*>(wring + static_cast<size_t>(p.slots) * p.blob_bytes);
    uint32_t* tbl = reinterpret_cast<uint32_t*>(red + 4 * TM * kTileN);  // mixed: the CTA's table entries
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const long long beg = unit_start(blockIdx.x, p.units, p.grid);
    const long long end = unit_start(blockIdx.x + 1, p.units, p.grid);
    if (threadIdx.x == 0) griddep_launch_dependents();
    if (warp == kWeightWarpR && lane == 0) prefetch_first_blobs<FMT == kFmtMixed>(p, beg, end);
    if (warp == 0) {
        for (int k = lane; k < kChunkBars; k += 32) mbar_init(&bars.full[k], 2);
        for (int s = lane; s < p.slots; s += 32) {
            mbar_init(&bars.empty_w[s], 4);  // the k-block's residue: 4 column-group warps
            mbar_init(&bars.empty_a[s], 4);
        }
        if (lane == 0) abort_flag = 0;
        if (FMT == kFmtMixed && lane == 0) mbar_init(&bars.tbl_full, 1);
        fence_barrier_init();
    }
    if (warp == kActWarpR && lane == 0)
        for (int c = 0; c < p.chunk; ++c) prefetch_tensor_map(&maps.m[c]);
    __syncthreads();

    const Ctl ctl{&abort_flag, p.status, p.timeout_ns};
    if (warp < kRfWarps) {
        if constexpr (is_group(MODE)) {
            if (p.scale_in_dequant)
                rf_role<MODE, TM, kRfScaleWeight, FMT>(p, aring, wring, bars, red, ctl, beg, end);
            else if (p.group_rows < kTileK)
                rf_role<MODE, TM, kRfScalePair, FMT>(p, aring, wring, bars, red, ctl, beg, end);
            else
                rf_role<MODE, TM, kRfScaleBlock, FMT>(p, aring, wring, bars, red, ctl, beg, end);
        } else {
            rf_role<MODE, TM, kRfScaleNone, FMT>(p, aring, wring, bars, red, ctl, beg, end);
        }
    } else if (warp == kWeightWarpR) {
        if constexpr (FMT == kFmtMixed) {
            long long tlo = 0;
            const bool tbl_ok = mixed_table_window(p, bars, tbl, ctl, beg, end, lane, &tlo);
            if (lane == 0) producer_role<MODE, true, true>(&maps, p, aring, wring, bars, ctl, beg, end, tbl, tlo, tbl_ok);
        } else {
            if (lane == 0) producer_role<MODE, true>(&maps, p, aring, wring, bars, ctl, beg, end);
        }
    } else {
        if (lane == 0) producer_role<MODE, false>(&maps, p, aring, wring, bars, ctl, beg, end);
    }
}

// ------------------------------------------------------------------ host side
// Bytes of the register-operand kernel's residue sums (after the ring in dynamic shared memory).
static int rf_red_bytes(int tm) { return 4 * tm * kTileN * 4; }

int make_plan(int mode, int M, int N, int K, int slots, int num_sms, int smem_optin, Plan* pl, int fmt) {
    pl->mode = mode;
    pl->k_blocks = K / kTileK;
    pl->n_tiles = n_tiles(N);
    const bool sparse = fmt == kFmtSparse;
    pl->sparse = sparse;
    pl->mixed = fmt == kFmtMixed;  // slots sized for the largest blob: every block 4-bit
    if (fmt != kFmtDense && (M > kRfMaxM || (mode != kModeGroup && mode != kModeChannel))) return -1;
    pl->blob_bytes = sparse                   ? static_cast<int>(blob_bytes_sp24(slots))
                     : (mode == kModeGroup)   ? static_cast<int>(blob_bytes_w4a16(slots))
                     : (mode == kModeGroupZP) ? static_cast<int>(blob_bytes_w4a16_zp(slots))
                                              : kCodeBytes;
    pl->rf = M <= kRfMaxM;
    if (pl->rf) {
        const int tm = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : (M <= 8 ? 8 : (M <= 16 ? 16 : 32))));
        pl->tile_m = tm;
        pl->m_tiles = 1;
        pl->small = false;
        pl->threads = kThreadsRf;
        pl->issuers = 0;
        // TM rows x 128 int8 or fp16, unswizzled; sparse: at least 8 rows, swizzled
        pl->act_rows = (sparse && tm < kSpMinActRows) ? kSpMinActRows : tm;
        pl->act_slot = (mode == kModeW4A8) ? tm * 128 : pl->act_rows * 256;
        // mixed: room for the CTA's table entries (at most ceil(units / grid) + 1 of them, widened to
        // 16-byte boundaries on both sides)
        const long long units = static_cast<long long>(pl->n_tiles) * pl->k_blocks;
        const long long per_cta = (units + num_sms - 1) / num_sms;
        const int tbl = pl->mixed ? static_cast<int>(((per_cta + 1 + 6) * 4 + 15) / 16 * 16) : 0;
        if (tbl > smem_optin) return -1;
        const int budget = smem_optin - 2048 - 1024 - rf_red_bytes(tm) - tbl;
        int s = budget / (pl->act_slot + pl->blob_bytes);
        if (s > kMaxSlots) s = kMaxSlots;
        if (s < 2) return -1;
        pl->slots = s;
        int c = s / 2;
        if (c > kMaxChunk) c = kMaxChunk;
        pl->chunk = c;
        pl->smem_bytes = s * (pl->act_slot + pl->blob_bytes) + 1024 + rf_red_bytes(tm) + tbl;
        pl->units = static_cast<long long>(pl->n_tiles) * pl->k_blocks;
        pl->grid = static_cast<int>(pl->units < num_sms ? pl->units : num_sms);
        return 0;
    }
    int mt = (M + kMaxTileM - 1) / kMaxTileM;
    if (mt < 1) mt = 1;
    int tm = (M + mt - 1) / mt;
    tm = ((tm + 15) / 16) * 16;
    if (tm < 16) tm = 16;
    pl->tile_m = tm;
    pl->act_rows = tm;
    pl->m_tiles = (M + tm - 1) / tm;
    if (pl->m_tiles < 1) pl->m_tiles = 1;
    pl->small = tm <= kSmallTileMax;
    pl->threads = pl->small ? kThreadsSmall : kThreadsLarge;
    pl->issuers = pl->small ? kMaxIssuers : (tm <= 64 ? 4 : (tm <= 128 ? 2 : 1));
    pl->act_slot = (mode == kModeW4A8) ? tm * 128 : tm * 256;
    const int budget = smem_optin - 2048 /* static shared memory */ - 1024 /* alignment slack */;
    int s = budget / (pl->act_slot + pl->blob_bytes);
    if (s > kMaxSlots) s = kMaxSlots;
    if (s < 2) return -1;
    pl->slots = s;
    int c = s / 2;
    if (c > kMaxChunk) c = kMaxChunk;
    if (c < 1) c = 1;
    pl->chunk = c;
    pl->smem_bytes = s * (pl->act_slot + pl->blob_bytes) + 1024;
    pl->units = static_cast<long long>(pl->n_tiles) * pl->m_tiles * pl->k_blocks;
    pl->grid = static_cast<int>(pl->units < num_sms ? pl->units : num_sms);
    return 0;
}

template <typename Kernel>
static cudaError_t allow_smem(Kernel k, int bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

cudaError_t configure_gemm_kernels(int max_dynamic_smem) {
    cudaError_t e = allow_smem(wq_gemm_large<kModeGroup>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_large<kModeChannel>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_large<kModeW4A8>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_small<kModeGroup, 32>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_small<kModeChannel, 32>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_small<kModeW4A8, 32>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_large<kModeGroupZP>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_small<kModeGroupZP, 32>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 1>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 2>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 4>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 1>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 2>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 4>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 1>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 2>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 4>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 8>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 8>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 8>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 1>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 2>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 4>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 8>, max_dynamic_smem);
    if constexpr (kRfMaxM > 8) {
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 16>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 16>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 16>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 16>, max_dynamic_smem);
    }
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 1, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 2, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 4, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 8, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 16, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 1, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 2, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 4, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 8, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 16, kFmtSparse>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 1, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 2, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 4, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 8, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 16, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 1, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 2, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 4, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 8, kFmtMixed>, max_dynamic_smem);
    if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 16, kFmtMixed>, max_dynamic_smem);
    if constexpr (kRfMaxM > 16) {
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroup, 32>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeChannel, 32>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeGroupZP, 32>, max_dynamic_smem);
        if (e == cudaSuccess) e = allow_smem(wq_gemm_rf<kModeW4A8, 32>, max_dynamic_smem);
    }
    return e;
}

template <typename Kernel>
static cudaError_t launch_kernel(Kernel k, const ActMaps& maps, const GemmArgs& args, const Plan& plan,
                                 cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid));
    cfg.blockDim = dim3(static_cast<unsigned>(plan.threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem_bytes);
    cfg.stream = st;
    // Programmatic dependent launch: a CTA may start on an SM that the previous kernel of the
    // stream has already left, set itself up and prefetch its first weights into L2 there.
    // No cooperative attribute: a cooperative grid is placed all at once, only after the
    // previous kernel has left every SM. The stream-K waits do not need it. A grid has at most
    // one CTA per SM and a CTA waits only for CTAs of lower index, so with CTAs dispatched in
    // index order every CTA waited for is resident, and the waits are bounded regardless.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, maps, args);
}

template <int MODE>
static cudaError_t launch_mode(const ActMaps& maps, const GemmArgs& args, const Plan& plan, cudaStream_t st) {
    {
        if (plan.rf && plan.sparse) {
            if constexpr (MODE == kModeGroup || MODE == kModeChannel) {
                if (plan.tile_m == 1) return launch_kernel(wq_gemm_rf<MODE, 1, kFmtSparse>, maps, args, plan, st);
                if (plan.tile_m == 2) return launch_kernel(wq_gemm_rf<MODE, 2, kFmtSparse>, maps, args, plan, st);
                if (plan.tile_m == 4) return launch_kernel(wq_gemm_rf<MODE, 4, kFmtSparse>, maps, args, plan, st);
                if (plan.tile_m == 8) return launch_kernel(wq_gemm_rf<MODE, 8, kFmtSparse>, maps, args, plan, st);
                if (plan.tile_m == 16) return launch_kernel(wq_gemm_rf<MODE, 16, kFmtSparse>, maps, args, plan, st);
            }
            return cudaErrorInvalidConfiguration;
        }
        if (plan.rf && plan.mixed) {
            if constexpr (MODE == kModeGroup || MODE == kModeChannel) {
                if (plan.tile_m == 1) return launch_kernel(wq_gemm_rf<MODE, 1, kFmtMixed>, maps, args, plan, st);
                if (plan.tile_m == 2) return launch_kernel(wq_gemm_rf<MODE, 2, kFmtMixed>, maps, args, plan, st);
                if (plan.tile_m == 4) return launch_kernel(wq_gemm_rf<MODE, 4, kFmtMixed>, maps, args, plan, st);
                if (plan.tile_m == 8) return launch_kernel(wq_gemm_rf<MODE, 8, kFmtMixed>, maps, args, plan, st);
                if (plan.tile_m == 16) return launch_kernel(wq_gemm_rf<MODE, 16, kFmtMixed>, maps, args, plan, st);
            }
            return cudaErrorInvalidConfiguration;
        }
        if (plan.sparse || plan.mixed) return cudaErrorInvalidConfiguration;
        if (plan.rf) {
            if (plan.tile_m == 1) return launch_kernel(wq_gemm_rf<MODE, 1>, maps, args, plan, st);
            if (plan.tile_m == 2) return launch_kernel(wq_gemm_rf<MODE, 2>, maps, args, plan, st);
            if (plan.tile_m == 4) return launch_kernel(wq_gemm_rf<MODE, 4>, maps, args, plan, st);
            if constexpr (kRfMaxM > 8) {
                if (plan.tile_m == 16) return launch_kernel(wq_gemm_rf<MODE, 16>, maps, args, plan, st);
            }
            if constexpr (kRfMaxM > 16) {
                if (plan.tile_m == 32) return launch_kernel(wq_gemm_rf<MODE, 32>, maps, args, plan, st);
            }
            return launch_kernel(wq_gemm_rf<MODE, 8>, maps, args, plan, st);
        }
    }
    if (!plan.small) return launch_kernel(wq_gemm_large<MODE>, maps, args, plan, st);
    // M <= 16 runs the register-operand kernel, so a small tile here is always 32 rows (M = 17..32)
    if (plan.tile_m != 32) return cudaErrorInvalidConfiguration;
    return launch_kernel(wq_gemm_small<MODE, 32>, maps, args, plan, st);
}

cudaError_t launch_gemm(int mode, const ActMaps& maps, const GemmArgs& args, const Plan& plan, cudaStream_t stream) {
    switch (mode) {
        case kModeGroup: return launch_mode<kModeGroup>(maps, args, plan, stream);
        case kModeChannel: return launch_mode<kModeChannel>(maps, args, plan, stream);
        case kModeGroupZP: return launch_mode<kModeGroupZP>(maps, args, plan, stream);
        default: return launch_mode<kModeW4A8>(maps, args, plan, stream);
    }
}

}  // namespace wq
