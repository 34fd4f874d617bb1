// Declarations shared by the library's translation units (not part of the public ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "wq_layout.h"

namespace wq {

// Arguments of the GEMM kernel (all three modes). Pointers are device pointers.
struct GemmArgs {
    const uint8_t* wp;         // prepacked blobs
    const uint16_t* s_chan;    // W4A16, g == K: fp16 column scales (n_tiles*128 entries)
    const float* sa;           // W4A8: per-token scales [M]
    const float* sw;           // W4A8: per-column scales [N]
    uint16_t* y;               // fp16 output [M, N]
    int32_t* acc_out;          // W4A8: optional int32 accumulators [M, N]
    float* ws_partial;         // stream-K partial tiles: [grid][tile_m][128] (fp32 or int32 bits)
    int* ws_flags;             // stream-K publish flags: [grid]
    int* status;               // device status word (0 = ok)
    int M, N;
    int m_tiles, n_tiles, k_blocks;
    int tile_m;                // MMA N extent (multiple of 16, <= 256)
    int issuers;               // MMA-issuing warps (1, 2 or 4); issuers * tile_m <= 256
    int slots;                 // shared-memory ring slots
    int chunk;                 // most k-blocks per copy
    int act_slot;              // bytes of one activation slot (one k-block of tile_m rows)
    int blob_bytes;            // bytes of one weight blob = one weight slot
    int group_rows;            // W4A16 grouped: rows per scale slot, min(g, 128)
    int small;                 // 1: per-k-block partials summed by the dequant warps (tile_m <= 32)
    int scale_in_dequant;      // 1: the dequant multiplies by the group scale (fp16 weights)
    int zp_offset;             // asymmetric groups: byte offset of the zero points within a blob
    const uint32_t* mix_table; // mixed 2/4-bit: the blob table at the start of wp (null otherwise)
    unsigned long long wp_bytes;  // mixed 2/4-bit: bytes of the caller's buffer (copies stay inside)
    long long units;           // tiles * k_blocks
    int grid;
    unsigned long long timeout_ns;
    int skip_publish;          // test hook: CTA that skips publishing its partial (-1: none)
};

// Activation tensor maps, one per chunk length 1..kMaxChunk (the box spans that many k-blocks).
struct ActMaps {
    CUtensorMap m[kMaxChunk];
};

struct Plan {
    int mode;
    int tile_m, m_tiles, n_tiles, k_blocks;
    long long units;
    int grid, issuers, slots, chunk, act_slot, blob_bytes, smem_bytes, threads;
    bool small;
    bool rf;    // M <= kRfMaxM: the register-operand kernel, unswizzled activation slots
    bool sparse;   // 2:4 sparse weights (register-operand kernel only; swizzled activation slots)
    bool mixed;    // mixed 2/4-bit weights (register-operand kernel only; blobs of varying size)
    int act_rows;  // rows of one activation copy: tile_m, or at least kSpMinActRows when sparse
};

// fmt: 0 dense, 1 2:4 sparse, 2 mixed 2/4-bit (the last two only for M <= kRfMaxM)
int make_plan(int mode, int M, int N, int K, int slots, int num_sms, int smem_optin, Plan* plan, int fmt = 0);

cudaError_t configure_gemm_kernels(int max_dynamic_smem);

cudaError_t launch_gemm(int mode, const ActMaps& maps, const GemmArgs& args, const Plan& plan,
                        cudaStream_t stream);

int launch_prepack(const int32_t* Q, const uint16_t* s, const uint8_t* z, int K, int N, int g, void* Wp,
                   cudaStream_t st);
int launch_prepack_w4a8(const int32_t* Q, int K, int N, void* Wp, cudaStream_t st);
int launch_unpack(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, uint8_t* z, cudaStream_t st);
int launch_unpack_w4a8(const void* Wp, int K, int N, int32_t* Q, cudaStream_t st);
int launch_prepack_sp24(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, int* bad,
                        cudaStream_t st);
int launch_unpack_sp24(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, cudaStream_t st);
int launch_prepack_mixed(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, int* bad, cudaStream_t st);
int launch_unpack_mixed(const void* Wp, int K, int N, int g, int32_t* Q, uint16_t* s, uint8_t* widths, cudaStream_t st);
int launch_quantize_act(const uint16_t* A, int M, int K, int bits, int8_t* Aq, float* sa, cudaStream_t st);
int launch_permute_codes(const int32_t* Q, const int32_t* perm, int K, int N, int32_t* Qp, cudaStream_t st);
int launch_permute_act(const uint16_t* A, const int32_t* perm, int M, int K, uint16_t* Ap, int* status,
                       cudaStream_t st);

}  // namespace wq
