// The mixed-precision linear layer on sm_100a: Y[M,N] = A[M,K] . dequant(Wp).
//
// What the pages ask of it ("MARLIN: Mixed-Precision Auto-Regressive Parallel Inference on
// Large Language Models", Abstract): stay memory-bound on the 4-bit weights over batch
// sizes 1..128 through asynchronous memory access, task scheduling, pipelining and bespoke
// quantisation support; hide the dequantisation ("Enabling Fast 2-bit LLM on GPUs: Memory
// Alignment and Asynchronous Dequantization", Abstract: dequantisation otherwise takes more
// than half of the run time). How this kernel does it on B200:
//
//   * The weights are the MMA's M operand (128 output columns per tile) and the activations
//     its N operand (tile_m rows, 16..256), so even M = 1 uses a legal tcgen05 shape.
//   * One persistent CTA per SM walks a contiguous range of (tile, k-block) units (stream-K).
//     A tile split between CTAs is finished by the CTA holding its last k-block, which adds
//     the other CTAs' fp32 partials in a fixed order: results are deterministic.
//   * Warp roles per CTA (320 threads):
//       warp 8      TMA producer: one bulk copy per weight blob (codes + scales, contiguous in
//                   HBM by construction of the prepack) and 2-D tensor copies of the
//                   activation tile (128-byte swizzle), into a ring of `stages` buffers;
//       warps 0..7  dequantisation: each thread owns one weight column of the tile (one
//                   tensor-memory lane) and half of the k-block; it turns 8 packed words into
//                   64 fp16 (or int8) values in registers and stores them into tensor memory,
//                   where they are the MMA's A operand: the dequantised weights never touch
//                   shared memory. The same warps run the epilogue;
//       warp 9      MMA issuer: tcgen05.mma with A from tensor memory, B (activations) from
//                   shared memory, accumulator in tensor memory; commits release the buffers.
//     Dequantisation of k-block i+1 overlaps the MMA of k-block i (4 tensor-memory slots).
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
    uint64_t full[kMaxStages];    // stage loaded (TMA transaction bytes)
    uint64_t empty[kMaxStages];   // stage consumed (8 dequant warps + 1 MMA commit)
    uint64_t afull[kASlots];      // dequantised weights in tensor memory (8 warps)
    uint64_t aempty[kASlots];     // MMA finished reading a tensor-memory slot (commit)
    uint64_t dfull;               // accumulator of a segment complete (commit)
    uint64_t drain;               // all MMAs of the CTA complete (commit)
};

struct Ctl {
    volatile int* abort_flag;     // shared: set by the first wait that gives up
    int* status;
    unsigned long long timeout_ns;
};

__device__ __forceinline__ void raise_error(const Ctl& c, int code) {
    *c.abort_flag = 1;
    atomicCAS(c.status, 0, code);
}

// Bounded wait on an mbarrier phase. Returns false when the CTA aborts or the limit expires.
__device__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c, bool honour_abort = true) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (honour_abort && *c.abort_flag) return false;
        if (global_timer_ns() - t0 > c.timeout_ns) {
            raise_error(c, WQ_ERR_TIMEOUT);
            return false;
        }
    }
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
        __nanosleep(100);
    }
}

// First unit of CTA c under the even split of `units` over `grid` CTAs.
__device__ __forceinline__ long long unit_start(int c, long long units, int grid) {
    return static_cast<long long>(c) * units / grid;
}

// Walks a CTA's unit range [beg, end) backwards, one segment (a run of k-blocks of one tile)
// at a time. Going backwards makes the CTA holding a tile's last k-block, which finishes the
// tile, the one that reaches that tile last, while the CTAs it waits for have lower indices
// and reach their part of the tile first.
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

// ------------------------------------------------------------------ dequantisation
// fp16 constants from the binary16 format: 0x6400 = 1024 (exponent field 25, so the 10
// mantissa bits count units), 0x6408 = 1032 = 1024 + 8, 0x2C00 = 1/16, 0xD480 = -72.
// (w & 0x000F000F) | 0x64006400 is the fp16 pair (1024 + q_lo, 1024 + q_hi) exactly;
// subtracting 1032 leaves q - 8 exactly. A nibble in bits 4..7 of a half gives 1024 + 16q;
// (1024 + 16q)/16 - 72 = q - 8, again exact in one fused multiply-add.
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

// int8 lanes 16*(q - 8): the code moved to the high nibble of its byte with the sign bit
// flipped ((q ^ 8) << 4) is 16*(q - 8) in two's complement. The accumulator is shifted
// right by 4 in the epilogue, exactly.
__device__ __forceinline__ void dequant_word_i8(uint32_t x, uint32_t* out) {
    out[0] = lop3_and_xor(x << 4, 0xF0F0F0F0u, 0x80808080u);  // codes 0..3 (low nibbles)
    out[1] = lop3_and_xor(x, 0xF0F0F0F0u, 0x80808080u);       // codes 4..7 (high nibbles)
}

// ------------------------------------------------------------------ epilogue
template <int MODE>
__device__ void epilogue(const GemmArgs& p, Barriers& b, uint32_t tmem, const Ctl& ctl, const SegCursor& seg,
                         int seg_index, int half, int quarter, int lane) {
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int nt = seg.tile / p.m_tiles, mt = seg.tile % p.m_tiles;
    const int n = nt * kTileN + row;
    const int cols = p.tile_m >> 1;
    const int c_begin = half * cols;
    const int m_base = mt * p.tile_m + c_begin;

    bool ok = __all_sync(0xffffffffu, wait_bar(&b.dfull, seg_index & 1, ctl));
    tc_fence_after();

    if (!seg.owner) {
        // contributor: publish this CTA's fp32 (or int32) partial tile, then raise its flag
        uint32_t* part = reinterpret_cast<uint32_t*>(p.ws_partial) + static_cast<size_t>(blockIdx.x) * p.tile_m * kTileN;
        for (int c = 0; c < cols; c += 8) {
            uint32_t v[8];
            if (ok) {
                tmem_ld_x8(tmem + lane_base + static_cast<uint32_t>(c_begin + c), v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 8; ++j) part[static_cast<size_t>(c_begin + c + j) * kTileN + row] = v[j];
            }
        }
        __threadfence();
        named_barrier_sync(1, kNumDqWarps * 32);
        if (threadIdx.x == 0 && ok && !*ctl.abort_flag && static_cast<int>(blockIdx.x) != p.skip_publish)
            st_release_gpu(&p.ws_flags[blockIdx.x], 1);
        return;
    }

    // owner: wait for the CTAs that hold the tile's lower k-blocks, nearest first
    const long long tbase = static_cast<long long>(seg.tile) * p.k_blocks;
    const int c_first = static_cast<int>(blockIdx.x) - 1;
    int c_last = c_first + 1;  // lowest contributing CTA index; c_first + 1 means none
    if (!seg.whole) {
        for (int c = c_first; c >= 0; --c) {
            c_last = c;
            if (ok) ok = wait_flag(&p.ws_flags[c], ctl);
            if (unit_start(c, p.units, p.grid) <= tbase) break;
        }
        ok = __all_sync(0xffffffffu, ok);
    }

    float s_col = 1.0f;
    if (MODE == kModeChannel) s_col = __half2float(__ushort_as_half(p.s_chan[n]));
    float sw_col = 0.0f;
    if (MODE == kModeW4A8) sw_col = n < p.N ? p.sw[n] : 0.0f;

    for (int c = 0; c < cols; c += 8) {
        uint32_t v[8];
        if (!ok) continue;
        tmem_ld_x8(tmem + lane_base + static_cast<uint32_t>(c_begin + c), v);
        tmem_ld_wait();
        for (int cc = c_first; cc >= c_last; --cc) {
            const uint32_t* part =
                reinterpret_cast<const uint32_t*>(p.ws_partial) + static_cast<size_t>(cc) * p.tile_m * kTileN;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t q = __ldcg(part + static_cast<size_t>(c_begin + c + j) * kTileN + row);
                if (MODE == kModeW4A8)
                    v[j] = static_cast<uint32_t>(static_cast<int32_t>(v[j]) + static_cast<int32_t>(q));
                else
                    v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(q));
            }
        }
        if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int m = m_base + c + j;
                if (m < p.M) {
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
    if (!seg.whole) {
        named_barrier_sync(1, kNumDqWarps * 32);
        if (threadIdx.x == 0)
            for (int cc = c_first; cc >= c_last; --cc) p.ws_flags[cc] = 0;  // ready for the next call
    }
}

// ------------------------------------------------------------------ roles
template <int MODE>
__device__ void dequant_role(const GemmArgs& p, uint8_t* smem, Barriers& b, uint32_t tmem, const Ctl& ctl,
                             long long beg, long long end) {
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;  // 128 k of fp16 or int8 per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t iter = 0;
    int seg_index = 0;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        for (int kb = seg.kb_hi; kb >= seg.kb_lo; --kb, ++iter) {
            const uint32_t s = iter % p.stages, ph = (iter / p.stages) & 1;
            const uint32_t a = iter % kASlots, aph = (iter / kASlots) & 1;
            bool ok = __all_sync(0xffffffffu, wait_bar(&b.full[s], ph, ctl));
            uint4 w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
            uint16_t sc0 = 0, sc1 = 0;
            if (ok) {
                const uint8_t* blob = smem + static_cast<size_t>(s) * p.stage_bytes + p.act_bytes;
                const uint4* words = reinterpret_cast<const uint4*>(blob);
                w0 = words[(half * 2 + 0) * kTileN + row];
                w1 = words[(half * 2 + 1) * kTileN + row];
                if (MODE == kModeGroup) {
                    const uint16_t* sc = reinterpret_cast<const uint16_t*>(blob + kCodeBytes);
                    sc0 = sc[((64 * half) / p.group_rows) * kTileN + row];
                    sc1 = sc[((64 * half + 32) / p.group_rows) * kTileN + row];
                }
            }
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(&b.empty[s]);
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
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dequant_word_f16(wv[i], i < 4 ? s0 : s1, MODE == kModeGroup, out + 4 * i);
                    tmem_st_x32(taddr, out);
                }
                tmem_st_wait();
                tc_fence_before();
            }
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(&b.afull[a]);
        }
        epilogue<MODE>(p, b, tmem, ctl, seg, seg_index, half, quarter, lane);
        ++seg_index;
    }
}

template <int MODE>
__device__ void producer_role(const CUtensorMap* tmap, const GemmArgs& p, uint8_t* smem, Barriers& b,
                              const Ctl& ctl, long long beg, long long end) {
    const uint64_t policy = l2_policy_evict_first();  // every weight byte is read once
    uint32_t iter = 0, issued = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        const int nt = seg.tile / p.m_tiles, mt = seg.tile % p.m_tiles;
        const uint8_t* wtile = p.wp + static_cast<size_t>(nt) * p.k_blocks * p.blob_bytes;
        const int y0 = mt * p.tile_m;
        for (int kb = seg.kb_hi; kb >= seg.kb_lo; --kb, ++iter) {
            const uint32_t s = iter % p.stages, ph = (iter / p.stages) & 1;
            if (ok) ok = wait_bar(&b.empty[s], ph ^ 1, ctl);
            if (!ok) continue;
            uint8_t* st = smem + static_cast<size_t>(s) * p.stage_bytes;
            mbar_arrive_expect_tx(&b.full[s], static_cast<uint32_t>(p.act_bytes + p.blob_bytes));
            if (MODE == kModeW4A8) {
                tma_load_2d(st, tmap, kb * kTileK, y0, &b.full[s]);
            } else {
                tma_load_2d(st, tmap, kb * kTileK, y0, &b.full[s]);
                tma_load_2d(st + p.tile_m * 128, tmap, kb * kTileK + 64, y0, &b.full[s]);
            }
            bulk_g2s(st + p.act_bytes, wtile + static_cast<size_t>(kb) * p.blob_bytes,
                     static_cast<uint32_t>(p.blob_bytes), &b.full[s], policy);
            issued = iter + 1;
        }
    }
    // wind-down: every copy this CTA started must land before the CTA exits
    const uint32_t n_stages = static_cast<uint32_t>(p.stages);
    for (uint32_t s = 0; s < n_stages && s < issued; ++s) {
        const uint32_t last = issued - 1 - ((issued - 1 - s) % n_stages);
        wait_bar(&b.full[s], (last / n_stages) & 1, ctl, false);
    }
}

template <int MODE>
__device__ void mma_role(const GemmArgs& p, uint8_t* smem, Barriers& b, uint32_t tmem, const Ctl& ctl,
                         long long beg, long long end) {
    constexpr int kSteps = (MODE == kModeW4A8) ? 4 : 8;          // MMA K: 32 int8 or 16 fp16
    constexpr int kSlotCols = (MODE == kModeW4A8) ? 32 : 64;
    const uint32_t idesc = (MODE == kModeW4A8) ? idesc_s8_s32(kTileN, p.tile_m) : idesc_f16_f32(kTileN, p.tile_m);
    const uint32_t smem_base = smem_addr(smem);
    uint32_t iter = 0;
    bool ok = true;
    SegCursor seg(beg, end, p.k_blocks);
    while (seg.next()) {
        for (int kb = seg.kb_hi; kb >= seg.kb_lo; --kb, ++iter) {
            const uint32_t s = iter % p.stages, ph = (iter / p.stages) & 1;
            const uint32_t a = iter % kASlots, aph = (iter / kASlots) & 1;
            if (ok) ok = wait_bar(&b.full[s], ph, ctl);
            if (ok) ok = wait_bar(&b.afull[a], aph, ctl);
            if (!ok) continue;
            tc_fence_after();
            const uint32_t act = smem_base + s * static_cast<uint32_t>(p.stage_bytes);
            const uint32_t a_tmem = tmem + kTmemAOffset + a * kSlotCols;
#pragma unroll
            for (int kk = 0; kk < kSteps; ++kk) {
                const uint32_t boff = (MODE == kModeW4A8)
                                          ? static_cast<uint32_t>(kk * 32)
                                          : static_cast<uint32_t>((kk >> 2) * p.tile_m * 128 + (kk & 3) * 32);
                const uint64_t bdesc = smem_desc_sw128(act + boff);
                const uint32_t accumulate = (kb != seg.kb_hi || kk != 0) ? 1u : 0u;
                if (MODE == kModeW4A8)
                    mma_i8_ts(tmem, a_tmem + kk * 8, bdesc, idesc, accumulate);
                else
                    mma_f16_ts(tmem, a_tmem + kk * 8, bdesc, idesc, accumulate);
            }
            tc_commit(&b.empty[s]);
            tc_commit(&b.aempty[a]);
        }
        if (ok) tc_commit(&b.dfull);
    }
    tc_commit(&b.drain);
    wait_bar(&b.drain, 0, ctl, false);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    wq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const GemmArgs p) {
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Barriers bars;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const uint32_t raw = smem_addr(smem_dyn);
    uint8_t* smem = smem_dyn + ((1024u - (raw & 1023u)) & 1023u);  // swizzle atoms need 1024-byte alignment
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], kNumDqWarps + 1);
        }
        for (int a = 0; a < kASlots; ++a) {
            mbar_init(&bars.afull[a], kNumDqWarps);
            mbar_init(&bars.aempty[a], 1);
        }
        mbar_init(&bars.dfull, 1);
        mbar_init(&bars.drain, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kTmaWarp && lane == 0) prefetch_tensor_map(&tmap_a);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const Ctl ctl{&abort_flag, p.status, p.timeout_ns};
    const long long beg = unit_start(blockIdx.x, p.units, p.grid);
    const long long end = unit_start(blockIdx.x + 1, p.units, p.grid);

    if (warp < kNumDqWarps) {
        dequant_role<MODE>(p, smem, bars, tmem, ctl, beg, end);
    } else if (warp == kTmaWarp) {
        if (lane == 0) producer_role<MODE>(&tmap_a, p, smem, bars, ctl, beg, end);
    } else {
        if (lane == 0) mma_role<MODE>(p, smem, bars, tmem, ctl, beg, end);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
int make_plan(int mode, int M, int N, int K, int slots, int num_sms, int smem_optin, Plan* pl) {
    pl->mode = mode;
    pl->k_blocks = K / kTileK;
    pl->n_tiles = n_tiles(N);
    int mt = (M + kMaxTileM - 1) / kMaxTileM;
    if (mt < 1) mt = 1;
    int tm = (M + mt - 1) / mt;
    tm = ((tm + 15) / 16) * 16;
    if (tm < 16) tm = 16;
    pl->tile_m = tm;
    pl->m_tiles = (M + tm - 1) / tm;
    if (pl->m_tiles < 1) pl->m_tiles = 1;
    pl->act_bytes = (mode == kModeW4A8) ? tm * 128 : tm * 256;
    pl->blob_bytes = (mode == kModeGroup) ? static_cast<int>(blob_bytes_w4a16(slots)) : kCodeBytes;
    pl->stage_bytes = (pl->act_bytes + pl->blob_bytes + 1023) / 1024 * 1024;
    const int budget = smem_optin - 2048 /* static shared memory */ - 1024 /* alignment slack */;
    int stages = budget / pl->stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return -1;
    pl->stages = stages;
    pl->smem_bytes = stages * pl->stage_bytes + 1024;
    pl->units = static_cast<long long>(pl->n_tiles) * pl->m_tiles * pl->k_blocks;
    pl->grid = static_cast<int>(pl->units < num_sms ? pl->units : num_sms);
    return 0;
}

cudaError_t configure_gemm_kernels(int max_dynamic_smem) {
    cudaError_t e = cudaFuncSetAttribute(wq_gemm_kernel<kModeGroup>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         max_dynamic_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(wq_gemm_kernel<kModeChannel>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_dynamic_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(wq_gemm_kernel<kModeW4A8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_dynamic_smem);
    return e;
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap& tmap, const GemmArgs& args, const Plan& plan, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem_bytes);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: the stream-K waits always end
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, wq_gemm_kernel<MODE>, tmap, args);
}

cudaError_t launch_gemm(int mode, const CUtensorMap& tmap, const GemmArgs& args, const Plan& plan,
                        cudaStream_t stream) {
    switch (mode) {
        case kModeGroup: return launch_mode<kModeGroup>(tmap, args, plan, stream);
        case kModeChannel: return launch_mode<kModeChannel>(tmap, args, plan, stream);
        default: return launch_mode<kModeW4A8>(tmap, args, plan, stream);
    }
}

}  // namespace wq
