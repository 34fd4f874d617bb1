// C ABI of the library (declared in include/wq.h): argument checks, launch plans, the
// per-(device, stream) stream-K workspace, tensor maps for the activation loads, and the
// device status word that reports expired waits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>
#include <utility>

#include "wq.h"
#include "wq_internal.h"

namespace {

using namespace wq;

constexpr int kVersion = 10000;  // 1.0.0
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
// W4A8 accumulates a * 16(q - 8) in int32; |a * 16(q - 8)| <= 128 * 128 = 16384 (a = -128,
// q = 0), and K * 16384 < 2^31 holds for every multiple of 128 up to 130944.
constexpr int kMaxKW4A8 = 130944;

std::mutex g_mu;
unsigned long long g_timeout_ns = kDefaultTimeoutNs;
int g_skip_publish = -1;

struct DeviceState {
    bool init = false;
    bool supported = false;
    int num_sms = 0;
    int smem_optin = 0;
    int* status = nullptr;  // device status word
    int* check = nullptr;   // 2:4 sparse layout pass: set when a group has more than two weights
};
std::map<int, DeviceState> g_devices;

struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
std::map<std::pair<int, uintptr_t>, Workspace> g_workspaces;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Initialise (once) and return the state of the current device; nullptr on CUDA failure.
DeviceState* device_state(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    *dev_out = dev;
    DeviceState& d = g_devices[dev];
    if (d.init) return &d;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return nullptr;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return nullptr;
    d.supported = (major == 10 && minor == 0);
    if (d.supported) {
        if (cudaMalloc(&d.status, sizeof(int)) != cudaSuccess) return nullptr;
        if (cudaMemset(d.status, 0, sizeof(int)) != cudaSuccess) return nullptr;
        if (cudaMalloc(&d.check, sizeof(int)) != cudaSuccess) return nullptr;
        if (configure_gemm_kernels(d.smem_optin - 2048) != cudaSuccess) return nullptr;
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return nullptr;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.init = true;
    return &d;
}

// Status of the current device for a compute call: WQ_OK with *out set, or an error.
int require_device(int* dev, DeviceState** out, cudaStream_t stream, bool need_init_outside_capture) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return WQ_ERR_CUDA;
    {
        int d = 0;
        if (cudaGetDevice(&d) != cudaSuccess) return WQ_ERR_CUDA;
        auto it = g_devices.find(d);
        if ((it == g_devices.end() || !it->second.init) && cs != cudaStreamCaptureStatusNone &&
            need_init_outside_capture)
            return WQ_ERR_CAPTURING;
    }
    DeviceState* st = device_state(dev);
    if (!st) return WQ_ERR_CUDA;
    if (!st->supported) return WQ_ERR_UNSUPPORTED_DEVICE;
    *out = st;
    return WQ_OK;
}

// Workspace of (dev, stream) with at least `bytes`; grows it (not while capturing).
int get_workspace(int dev, cudaStream_t stream, size_t bytes, void** ptr) {
    Workspace& w = g_workspaces[{dev, reinterpret_cast<uintptr_t>(stream)}];
    if (w.bytes >= bytes && w.ptr) {
        *ptr = w.ptr;
        return WQ_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return WQ_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return WQ_ERR_CAPTURING;
    size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
    if (w.ptr) {
        if (cudaStreamSynchronize(stream) != cudaSuccess) return WQ_ERR_CUDA;
        cudaFree(w.ptr);
        w.ptr = nullptr;
        w.bytes = 0;
    }
    if (cudaMalloc(&w.ptr, want) != cudaSuccess) {
        cudaGetLastError();
        w.ptr = nullptr;
        return WQ_ERR_NO_MEMORY;
    }
    if (cudaMemsetAsync(w.ptr, 0, want, stream) != cudaSuccess) return WQ_ERR_CUDA;
    w.bytes = want;
    *ptr = w.ptr;
    return WQ_OK;
}

// Layout of a workspace: flags [grid] int32 at offset 0, partial tiles from offset 4096 on.
// 1 when the dequant multiplies the group scale into the fp16 weight (one rounding per weight):
// large tiles always; small tiles for g = 32, 64 (g >= 128 scales each k-block's fp32 partial);
// register-operand tiles for g = 32 (g >= 64 scales each k-block's fp32 sum).
int scale_in_dequant(const Plan& pl, int g) {
    if (pl.mode != kModeGroup && pl.mode != kModeGroupZP) return 0;
    if (pl.rf) return g < 64 ? 1 : 0;
    return (!pl.small || g < kTileK) ? 1 : 0;
}

size_t workspace_bytes_for(const Plan& pl) {
    return 4096 + static_cast<size_t>(pl.grid) * pl.tile_m * kTileN * 4;
}

// kind 0: W4A16; 1: W4A8; 3: W4A16 with a zero point per group (g < K); 5: 2:4 sparse W4A16;
// 6: mixed 2/4-bit W4A16 (5 and 6: M <= kRfMaxM).
int plan_for(int kind, int M, int N, int K, int g, const DeviceState& d, Plan* pl) {
    int mode;
    int slots = 0;
    if (kind == 0 || kind == 3 || kind == 5 || kind == 6) {
        slots = scale_slots(K, g);
        if (slots < 0 || (kind == 3 && slots == 0)) return WQ_ERR_INVALID_ARG;
        mode = kind == 3 ? kModeGroupZP : (slots > 0 ? kModeGroup : kModeChannel);
    } else {
        mode = kModeW4A8;
    }
    if ((kind == 5 || kind == 6) && M > kRfMaxM) return WQ_ERR_UNSUPPORTED_SHAPE;
    const int fmt = kind == 5 ? 1 : (kind == 6 ? 2 : 0);
    if (make_plan(mode, M, N, K, slots, d.num_sms, d.smem_optin, pl, fmt) != 0) return WQ_ERR_UNSUPPORTED_SHAPE;
    return WQ_OK;
}

// Activation maps for chunks of 1..chunk k-blocks. A [M, K] is seen as 3-D with the k-block
// split into swizzle-wide pieces: dims {64 fp16 or 128 int8, M, K/piece}, strides {K*elem (rows),
// piece bytes}; a box of {piece, tile_m, c*pieces_per_kblock} lands in shared memory as
// [piece index][row][128 bytes], the K-major 128-byte-swizzled layout the MMA reads.
// Unswizzled (swizzle false: the register-operand kernel on dense weights) the box lands as
// [piece][row][64 fp16]. tile_m is the box's row count (rows past M read as zeros).
int encode_activation_maps(ActMaps* maps, const void* A, int M, int K, int tile_m, int chunk, bool int8,
                           bool swizzle = true) {
    const int piece = int8 ? 128 : 64;                 // elements per 128-byte row
    const int per_kblock = kTileK / piece;             // 1 (int8) or 2 (fp16)
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(piece), static_cast<cuuint64_t>(M),
                                static_cast<cuuint64_t>(K / piece)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * (int8 ? 1u : 2u), 128u};
    const cuuint32_t estr[3] = {1, 1, 1};
    std::memset(maps, 0, sizeof(*maps));
    for (int c = 1; c <= chunk; ++c) {
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(piece), static_cast<cuuint32_t>(tile_m),
                                   static_cast<cuuint32_t>(c * per_kblock)};
        CUresult r = g_encode(&maps->m[c - 1], int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                              const_cast<void*>(A), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int check_shape(int K, int N) {
    if (K <= 0 || N <= 0) return WQ_ERR_INVALID_ARG;
    if (!shape_ok(K, N)) return WQ_ERR_UNSUPPORTED_SHAPE;
    return WQ_OK;
}

// Bytes of the activation buffers the W4A8 call with fp16 activations keeps in the workspace
// after the stream-K part: int8 codes [M, K] and fp32 scales [M], each 256-byte aligned.
size_t act_quant_bytes(int M, int K) {
    return ((static_cast<size_t>(M) * K + 255) / 256) * 256 + ((static_cast<size_t>(M) * 4 + 255) / 256) * 256;
}

// Bytes of the gathered activations the act-order call keeps in the workspace after the
// stream-K part: fp16 [M, K], 256-byte aligned.
size_t act_perm_bytes(int M, int K) { return ((static_cast<size_t>(M) * K * 2 + 255) / 256) * 256; }

// Act-order gathers launch M * ceil(K / 2048) CTAs; the grid must stay below 2^31.
bool perm_grid_ok(int M, int K) {
    return static_cast<long long>(M) * ((K / 8 + 255) / 256) < (1LL << 31) - 1;
}

// The W4A16 (kind 0), W4A8 (kind 1), zero-point (kind 3), 2:4 sparse (kind 5) or mixed 2/4-bit
// (kind 6) layer. A_fp16 (W4A8 only, may be
// null): fp16 activations that are first quantised per token into the workspace (the codes
// replace A, the scales go to sa_out when given, else to the workspace). perm (kinds 0 and 3,
// may be null): act order; A's columns are first gathered in the order perm into the
// workspace, which then replaces A.
int run_gemm(int kind, const void* A, const float* sa, const void* Wp, const float* sw, uint16_t* Y,
             int32_t* acc_out, int M, int N, int K, int g, cudaStream_t stream, const uint16_t* A_fp16 = nullptr,
             float* sa_out = nullptr, int act_bits = 8, const int32_t* perm = nullptr, size_t wp_bytes = 0) {
    int rc = check_shape(K, N);
    if (rc) return rc;
    if (M < 0) return WQ_ERR_INVALID_ARG;
    if (M > (1 << 24)) return WQ_ERR_UNSUPPORTED_SHAPE;
    if ((kind == 0 || kind == 3 || kind == 5 || kind == 6) && scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (kind == 3 && scale_slots(K, g) == 0) return WQ_ERR_INVALID_ARG;
    if ((kind == 5 || kind == 6) && M > kRfMaxM) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (kind == 1 && K > kMaxKW4A8) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (kind == 6 && wp_bytes < wq_prepacked_bytes_mixed(K, N, g, 0)) return WQ_ERR_INVALID_ARG;
    if (!Wp) return WQ_ERR_INVALID_ARG;
    if (!aligned(Wp, 16)) return WQ_ERR_MISALIGNED;
    if (M == 0) return WQ_OK;
    if (A_fp16) {
        if (!Y || !sw) return WQ_ERR_INVALID_ARG;
        if (!aligned(A_fp16, 16) || (sa_out && !aligned(sa_out, 4))) return WQ_ERR_MISALIGNED;
    } else {
        if (!A || !Y || (kind == 1 && (!sa || !sw))) return WQ_ERR_INVALID_ARG;
        if (!aligned(A, 16) || (kind == 1 && !aligned(sa, 4))) return WQ_ERR_MISALIGNED;
    }
    if (!aligned(Y, 16) || (acc_out && !aligned(acc_out, 16))) return WQ_ERR_MISALIGNED;
    if (kind == 1 && !aligned(sw, 4)) return WQ_ERR_MISALIGNED;
    if (perm && !aligned(perm, 16)) return WQ_ERR_MISALIGNED;
    if (perm && !perm_grid_ok(M, K)) return WQ_ERR_UNSUPPORTED_SHAPE;

    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, stream, true);
    if (rc) return rc;
    Plan pl;
    rc = plan_for(kind, M, N, K, g, *d, &pl);
    if (rc) return rc;
    void* ws = nullptr;
    const size_t gemm_ws = (workspace_bytes_for(pl) + 255) / 256 * 256;
    rc = get_workspace(dev, stream,
                       gemm_ws + (A_fp16 ? act_quant_bytes(M, K) : 0) + (perm ? act_perm_bytes(M, K) : 0), &ws);
    if (rc) return rc;
    if (perm) {
        uint16_t* Ap = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + gemm_ws);
        if (launch_permute_act(static_cast<const uint16_t*>(A), perm, M, K, Ap, d->status, stream) != 0) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
        A = Ap;
    }
    if (A_fp16) {
        int8_t* Aq = reinterpret_cast<int8_t*>(static_cast<uint8_t*>(ws) + gemm_ws);
        float* sq = sa_out ? sa_out
                           : reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + gemm_ws +
                                                      (static_cast<size_t>(M) * K + 255) / 256 * 256);
        if (launch_quantize_act(A_fp16, M, K, act_bits, Aq, sq, stream) != 0) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
        A = Aq;
        sa = sq;
    }
    ActMaps maps;
    rc = encode_activation_maps(&maps, A, M, K, pl.act_rows, pl.chunk, kind == 1, !pl.rf || pl.sparse);
    if (rc) return rc;

    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.wp = static_cast<const uint8_t*>(Wp);
    const long long nblob = static_cast<long long>(pl.n_tiles) * pl.k_blocks;
    a.s_chan = (pl.mode != kModeChannel) ? nullptr
               : reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(Wp) +
                                                   (pl.mixed ? mixed_table_bytes(nblob)
                                                             : static_cast<size_t>(nblob) * pl.blob_bytes));
    a.mix_table = pl.mixed ? static_cast<const uint32_t*>(Wp) : nullptr;
    a.wp_bytes = wp_bytes;
    a.sa = sa;
    a.sw = sw;
    a.y = Y;
    a.acc_out = acc_out;
    a.ws_flags = static_cast<int*>(ws);
    a.ws_partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 4096);
    a.status = d->status;
    a.M = M;
    a.N = N;
    a.m_tiles = pl.m_tiles;
    a.n_tiles = pl.n_tiles;
    a.k_blocks = pl.k_blocks;
    a.tile_m = pl.tile_m;
    a.issuers = pl.issuers;
    a.slots = pl.slots;
    a.chunk = pl.chunk;
    a.act_slot = pl.act_slot;
    a.blob_bytes = pl.blob_bytes;
    a.group_rows = ((kind == 0 || kind == 3 || kind == 5 || kind == 6) && g < kTileK) ? g : kTileK;
    a.small = pl.small ? 1 : 0;
    a.scale_in_dequant = scale_in_dequant(pl, g);
    a.zp_offset = (pl.mode == kModeGroupZP) ? static_cast<int>(blob_bytes_w4a16(scale_slots(K, g))) : 0;
    a.units = pl.units;
    a.grid = pl.grid;
    a.timeout_ns = g_timeout_ns;
    a.skip_publish = g_skip_publish;
    if (launch_gemm(pl.mode, maps, a, pl, stream) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int prepack_common_checks(const void* Q, int K, int N, const void* Wp, cudaStream_t stream) {
    int rc = check_shape(K, N);
    if (rc) return rc;
    if (!Q || !Wp) return WQ_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(Wp, 16)) return WQ_ERR_MISALIGNED;
    (void)stream;
    return WQ_OK;
}

}  // namespace

// ---------------------------------------------------------------- fixed-scratch W4A16 call
// Some callers cannot call cudaMalloc at the point where they run the layer: an engine that
// hands all free device memory to its own pool (KV cache, activations) at start-up and must
// not see outside allocations fail or fragment it; a plugin whose host framework owns every
// allocation; a latency-critical loop that must not risk the implicit synchronisation of an
// allocation. wq_gemm_w4a16 grows a per-(device, stream) workspace with cudaMalloc on first
// use; wq_gemm_w4a16_noalloc runs the same kernels with their stream-K scratch (publish flags
// and partial tiles) in the fixed array below instead, which the CUDA module loader sets
// aside on every device that loads this library, for the life of the process.
//
// Layout: flags int32 [grid] at offset 0 (must be zero at launch; cleared by every call),
// partial tiles from offset 4096, the kernels' status word in the last 256 bytes.
constexpr size_t kNoAllocScratchBytes = WQ_NOALLOC_SCRATCH_BYTES;
constexpr size_t kNoAllocStatusOffset = kNoAllocScratchBytes - 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxDevices = 64;

struct NoAllocDevice {
    bool ready = false;
    int num_sms = 0;
    int smem_optin = 0;
    unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocDevice g_noalloc[kNoAllocMaxDevices];

// One-time set-up of the current device for the fixed-scratch call: no allocation, only
// attribute queries, kernel attributes, the symbol's device address and two blocking clears.
int noalloc_device(int* dev_out, NoAllocDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return WQ_ERR_UNSUPPORTED_DEVICE;
    NoAllocDevice& d = g_noalloc[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return WQ_ERR_CUDA;
        if (major != 10 || minor != 0) return WQ_ERR_UNSUPPORTED_DEVICE;
        if (configure_gemm_kernels(d.smem_optin - 2048) != cudaSuccess) return WQ_ERR_CUDA;
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return WQ_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        // host code must not use g_noalloc_scratch itself: on the host it names a stand-in
        // object, not device memory. The device address is per device, taken with it current.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
        unsigned char* base = static_cast<unsigned char*>(p);
        if (cudaMemset(base, 0, 4096) != cudaSuccess) return WQ_ERR_CUDA;
        if (cudaMemset(base + kNoAllocStatusOffset, 0, 256) != cudaSuccess) return WQ_ERR_CUDA;
        d.scratch = base;
        d.ready = true;
    }
    *dev_out = dev;
    *out = &d;
    return WQ_OK;
}

}  // namespace

extern "C" {

const char* wq_status_string(int status) {
    switch (status) {
        case WQ_OK: return "WQ_OK";
        case WQ_ERR_INVALID_ARG: return "WQ_ERR_INVALID_ARG: null pointer, negative size or unsupported group size";
        case WQ_ERR_UNSUPPORTED_SHAPE:
            return "WQ_ERR_UNSUPPORTED_SHAPE: K must be a multiple of 128, N a multiple of 8, M at most 2^24 "
                   "(2:4 sparse and mixed 2/4-bit weights: M at most 16)";
        case WQ_ERR_MISALIGNED: return "WQ_ERR_MISALIGNED: a pointer breaks the alignment rule";
        case WQ_ERR_UNSUPPORTED_DEVICE: return "WQ_ERR_UNSUPPORTED_DEVICE: needs compute capability 10.0 (sm_100a)";
        case WQ_ERR_CUDA: return "WQ_ERR_CUDA: a CUDA call or kernel launch failed";
        case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT: a device-side wait expired";
        case WQ_ERR_NO_MEMORY: return "WQ_ERR_NO_MEMORY: workspace allocation failed";
        case WQ_ERR_CAPTURING: return "WQ_ERR_CAPTURING: reserve the workspace before capturing the stream";
        case WQ_ERR_NOT_SPARSE:
            return "WQ_ERR_NOT_SPARSE: a run of 4 weight rows holds more than 2 codes other than 8";
        case WQ_ERR_SCRATCH_LIMIT:
            return "WQ_ERR_SCRATCH_LIMIT: the call needs more stream-K scratch than the fixed array of "
                   "wq_gemm_w4a16_noalloc holds (use wq_gemm_w4a16)";
        default: return "WQ_ERR_UNKNOWN";
    }
}

int wq_version(void) { return kVersion; }

size_t wq_prepacked_bytes(int K, int N, int g) {
    if (!shape_ok(K, N)) return 0;
    const int slots = scale_slots(K, g);
    if (slots < 0) return 0;
    const size_t nblob = static_cast<size_t>(n_tiles(N)) * (K / kTileK);
    if (slots == 0) return nblob * kCodeBytes + channel_tail_bytes(N);
    return nblob * blob_bytes_w4a16(slots);
}

size_t wq_prepacked_bytes_w4a8(int K, int N) {
    if (!shape_ok(K, N)) return 0;
    return static_cast<size_t>(n_tiles(N)) * (K / kTileK) * kCodeBytes;
}

int wq_prepack(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (!s) return WQ_ERR_INVALID_ARG;
    if (!aligned(s, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_prepack(Q, s, nullptr, K, N, g, Wp, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_prepack_w4a8(const int32_t* Q, int K, int N, void* Wp, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_prepack_w4a8(Q, K, N, Wp, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_unpack(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q_out, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (!s_out) return WQ_ERR_INVALID_ARG;
    if (!aligned(s_out, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_unpack(Wp, K, N, g, Q_out, s_out, nullptr, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_unpack_w4a8(const void* Wp, int K, int N, int32_t* Q_out, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q_out, K, N, Wp, st);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_unpack_w4a8(Wp, K, N, Q_out, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a16(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g, void* stream) {
    return run_gemm(0, A, nullptr, Wp, nullptr, Y, nullptr, M, N, K, g, static_cast<cudaStream_t>(stream));
}

size_t wq_prepacked_bytes_zp(int K, int N, int g) {
    if (!shape_ok(K, N)) return 0;
    const int slots = scale_slots(K, g);
    if (slots <= 0) return 0;
    return static_cast<size_t>(n_tiles(N)) * (K / kTileK) * blob_bytes_w4a16_zp(slots);
}

int wq_prepack_zp(const int32_t* Q, const uint16_t* s, const uint8_t* z, int K, int N, int g, void* Wp, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) <= 0) return WQ_ERR_INVALID_ARG;
    if (!s || !z) return WQ_ERR_INVALID_ARG;
    if (!aligned(s, 16) || !aligned(z, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_prepack(Q, s, z, K, N, g, Wp, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_unpack_zp(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, uint8_t* z_out, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q_out, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) <= 0) return WQ_ERR_INVALID_ARG;
    if (!s_out || !z_out) return WQ_ERR_INVALID_ARG;
    if (!aligned(s_out, 16) || !aligned(z_out, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_unpack(Wp, K, N, g, Q_out, s_out, z_out, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a16_zp(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g, void* stream) {
    return run_gemm(3, A, nullptr, Wp, nullptr, Y, nullptr, M, N, K, g, static_cast<cudaStream_t>(stream));
}

int wq_prepack_act_order(const int32_t* Q, const uint16_t* s, const uint8_t* z, const int32_t* perm, int K, int N,
                         int g, void* Wp, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    const int slots = scale_slots(K, g);
    if (slots < 0 || (z && slots == 0)) return WQ_ERR_INVALID_ARG;
    if (!s || !perm) return WQ_ERR_INVALID_ARG;
    if (!aligned(s, 16) || !aligned(perm, 16) || (z && !aligned(z, 16))) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    // perm must be a permutation of 0..K-1: checked on the host (once per weight), so the
    // reordering kernel never reads outside Q
    std::vector<int32_t> h(static_cast<size_t>(K));
    if (cudaMemcpyAsync(h.data(), perm, h.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    std::vector<char> seen(static_cast<size_t>(K), 0);
    for (int32_t r : h) {
        if (r < 0 || r >= K || seen[r]) return WQ_ERR_INVALID_ARG;
        seen[r] = 1;
    }
    void* Qp = nullptr;
    if (cudaMallocAsync(&Qp, static_cast<size_t>(K / 8) * N * sizeof(int32_t), st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_NO_MEMORY;
    }
    rc = WQ_OK;
    if (launch_permute_codes(Q, perm, K, N, static_cast<int32_t*>(Qp), st) != 0 ||
        launch_prepack(static_cast<const int32_t*>(Qp), s, z, K, N, g, Wp, st) != 0) {
        cudaGetLastError();
        rc = WQ_ERR_CUDA;
    }
    if (cudaFreeAsync(Qp, st) != cudaSuccess) {
        cudaGetLastError();
        rc = WQ_ERR_CUDA;
    }
    return rc;
}

int wq_permute_act(const uint16_t* A, const int32_t* perm, int M, int K, uint16_t* A_out, void* stream) {
    if (K <= 0 || M < 0) return WQ_ERR_INVALID_ARG;
    if (K % 8 || M > (1 << 24) || !perm_grid_ok(M, K)) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return WQ_OK;
    if (!A || !perm || !A_out) return WQ_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(perm, 16) || !aligned(A_out, 16)) return WQ_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    int rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_permute_act(A, perm, M, K, A_out, d->status, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a16_act_order(const uint16_t* A, const int32_t* perm, const void* Wp, uint16_t* Y, int M, int N,
                            int K, int g, int zero_points, void* stream) {
    if (M > 0 && (!A || !perm)) return WQ_ERR_INVALID_ARG;
    if (zero_points != 0 && zero_points != 1) return WQ_ERR_INVALID_ARG;
    return run_gemm(zero_points ? 3 : 0, A, nullptr, Wp, nullptr, Y, nullptr, M, N, K, g,
                    static_cast<cudaStream_t>(stream), nullptr, nullptr, 8, perm);
}

size_t wq_prepacked_bytes_sparse24(int K, int N, int g) {
    if (!shape_ok(K, N)) return 0;
    const int slots = scale_slots(K, g);
    if (slots < 0) return 0;
    const size_t nblob = static_cast<size_t>(n_tiles(N)) * (K / kTileK);
    if (slots == 0) return nblob * blob_bytes_sp24(0) + channel_tail_bytes(N);
    return nblob * blob_bytes_sp24(slots);
}

int wq_prepack_sparse24(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (!s) return WQ_ERR_INVALID_ARG;
    if (!aligned(s, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return WQ_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return WQ_ERR_CAPTURING;  // the check below synchronises
    int bad = 0;
    if (cudaMemsetAsync(d->check, 0, sizeof(int), st) != cudaSuccess ||
        launch_prepack_sp24(Q, s, K, N, g, Wp, d->check, st) != 0 ||
        cudaMemcpyAsync(&bad, d->check, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return bad ? WQ_ERR_NOT_SPARSE : WQ_OK;
}

int wq_unpack_sparse24(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q_out, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (!s_out) return WQ_ERR_INVALID_ARG;
    if (!aligned(s_out, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_unpack_sp24(Wp, K, N, g, Q_out, s_out, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a16_sparse24(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g, void* stream) {
    return run_gemm(5, A, nullptr, Wp, nullptr, Y, nullptr, M, N, K, g, static_cast<cudaStream_t>(stream));
}

size_t wq_prepacked_bytes_mixed(int K, int N, int g, long long n4) {
    if (!shape_ok(K, N)) return 0;
    const int slots = scale_slots(K, g);
    if (slots < 0) return 0;
    const long long nblob = static_cast<long long>(n_tiles(N)) * (K / kTileK);
    if (n4 < 0 || n4 > 4 * nblob) return 0;
    return mixed_table_bytes(nblob) + (slots ? 0 : channel_tail_bytes(N)) + static_cast<size_t>(4 * nblob + n4) * kMixBlock2 +
           static_cast<size_t>(nblob) * 2 * kTileN * slots;
}

int wq_prepack_mixed(const int32_t* Q, const uint16_t* s, const uint8_t* widths, int K, int N, int g, void* Wp,
                     size_t wp_bytes, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q, K, N, Wp, st);
    if (rc) return rc;
    const int slots = scale_slots(K, g);
    if (slots < 0 || !s || !widths) return WQ_ERR_INVALID_ARG;
    if (!aligned(s, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return WQ_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return WQ_ERR_CAPTURING;  // the widths are read on the host
    const int KT = K / kTileK, NT = n_tiles(N);
    const long long nblob = static_cast<long long>(NT) * KT;
    std::vector<uint8_t> w(static_cast<size_t>(K / kMixBlockRows) * NT);
    if (cudaMemcpyAsync(w.data(), widths, w.size(), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    // the blob table: each blob's offset (a prefix sum over the widths) and its widths
    std::vector<uint32_t> table(mixed_table_bytes(nblob) / 4, 0u);  // the padding written as zeros too
    size_t pos = mixed_table_bytes(nblob) + (slots ? 0 : channel_tail_bytes(N));
    for (int nt = 0; nt < NT; ++nt)
        for (int kt = 0; kt < KT; ++kt) {
            uint32_t wbits = 0;
            for (int v = 0; v < 4; ++v) {
                const uint8_t x = w[static_cast<size_t>(kt * 4 + v) * NT + nt];
                if (x != 2 && x != 4) return WQ_ERR_INVALID_ARG;
                if (x == 4) wbits |= 1u << v;
            }
            if (pos / 16 >= (1u << 28)) return WQ_ERR_UNSUPPORTED_SHAPE;  // 28 bits of offset per entry
            table[static_cast<size_t>(nt) * KT + kt] = static_cast<uint32_t>(pos / 16) << 4 | wbits;
            pos += static_cast<size_t>(kMixBlock2) * (4 + __builtin_popcount(wbits)) + 2 * kTileN * slots;
        }
    if (pos / 16 >= (1u << 28)) return WQ_ERR_UNSUPPORTED_SHAPE;
    table[static_cast<size_t>(nblob)] = static_cast<uint32_t>(pos / 16) << 4;
    if (pos > wp_bytes) return WQ_ERR_INVALID_ARG;  // the caller's buffer is smaller than the format needs
    int bad = 0;
    if (cudaMemcpyAsync(Wp, table.data(), table.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemsetAsync(d->check, 0, sizeof(int), st) != cudaSuccess ||
        launch_prepack_mixed(Q, s, K, N, g, Wp, d->check, st) != 0 ||
        cudaMemcpyAsync(&bad, d->check, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return bad ? WQ_ERR_INVALID_ARG : WQ_OK;
}

int wq_unpack_mixed(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, uint8_t* widths_out,
                    void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = prepack_common_checks(Q_out, K, N, Wp, st);
    if (rc) return rc;
    if (scale_slots(K, g) < 0 || !s_out || !widths_out) return WQ_ERR_INVALID_ARG;
    if (!aligned(s_out, 16)) return WQ_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_unpack_mixed(Wp, K, N, g, Q_out, s_out, widths_out, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a16_mixed(const uint16_t* A, const void* Wp, size_t wp_bytes, uint16_t* Y, int M, int N, int K, int g,
                        void* stream) {
    return run_gemm(6, A, nullptr, Wp, nullptr, Y, nullptr, M, N, K, g, static_cast<cudaStream_t>(stream), nullptr,
                    nullptr, 8, nullptr, wp_bytes);
}

int wq_gemm_w4a8(const int8_t* A, const float* sa, const void* Wp, const float* sw, uint16_t* Y, int32_t* acc_out,
                 int M, int N, int K, void* stream) {
    return run_gemm(1, A, sa, Wp, sw, Y, acc_out, M, N, K, K, static_cast<cudaStream_t>(stream));
}

int wq_quantize_act(const uint16_t* A, int M, int K, int bits, int8_t* A_q, float* sa, void* stream) {
    if (K <= 0 || M < 0 || (bits != 4 && bits != 8)) return WQ_ERR_INVALID_ARG;
    if (K % 8 || M > (1 << 24)) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return WQ_OK;
    if (!A || !A_q || !sa) return WQ_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(A_q, 16) || !aligned(sa, 4)) return WQ_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    int rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    if (launch_quantize_act(A, M, K, bits, A_q, sa, st) != 0) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

int wq_gemm_w4a8_fp16act(const uint16_t* A, const void* Wp, const float* sw, uint16_t* Y, int32_t* acc_out,
                         float* sa_out, int M, int N, int K, int act_bits, void* stream) {
    if ((M > 0 && !A) || (act_bits != 4 && act_bits != 8)) return WQ_ERR_INVALID_ARG;
    return run_gemm(1, nullptr, nullptr, Wp, sw, Y, acc_out, M, N, K, K, static_cast<cudaStream_t>(stream), A,
                    sa_out, act_bits);
}

size_t wq_workspace_bytes(int kind, int M, int N, int K) {
    if (!shape_ok(K, N) || M <= 0 || kind < 0 || kind > 6) return 0;
    if ((kind == 5 || kind == 6) && M > kRfMaxM) return 0;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = device_state(&dev);
    if (!d || !d->supported) return 0;
    Plan pl;
    const bool w4a16 = kind == 0 || kind >= 3;  // these plan like the W4A16 layer
    if (plan_for(w4a16 ? 0 : 1, M, N, K, w4a16 ? kTileK : K, *d, &pl) != WQ_OK) return 0;
    if (kind == 2) return (workspace_bytes_for(pl) + 255) / 256 * 256 + act_quant_bytes(M, K);
    if (kind == 4) return (workspace_bytes_for(pl) + 255) / 256 * 256 + act_perm_bytes(M, K);
    return workspace_bytes_for(pl);
}

int wq_workspace_reserve(size_t bytes, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    int rc = require_device(&dev, &d, st, true);
    if (rc) return rc;
    void* p = nullptr;
    return get_workspace(dev, st, bytes, &p);
}

int wq_get_device_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    DeviceState* d = nullptr;
    int rc = require_device(&dev, &d, st, false);
    if (rc) return rc;
    if (cudaStreamSynchronize(st) != cudaSuccess) return WQ_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WQ_ERR_CUDA;
    // the fixed-scratch call keeps its own status word in its array (read and cleared here
    // without any allocation)
    int h_fixed = 0;
    NoAllocDevice* na = (dev >= 0 && dev < kNoAllocMaxDevices && g_noalloc[dev].ready) ? &g_noalloc[dev] : nullptr;
    if (na && cudaMemcpy(&h_fixed, na->scratch + kNoAllocStatusOffset, sizeof(int), cudaMemcpyDeviceToHost) !=
                  cudaSuccess)
        return WQ_ERR_CUDA;
    if (h == WQ_OK && h_fixed == WQ_OK) return WQ_OK;
    // a wait expired: clear the status words and every workspace's flags of this device
    if (h != WQ_OK) {
        if (cudaMemset(d->status, 0, sizeof(int)) != cudaSuccess) return WQ_ERR_CUDA;
        for (auto& kv : g_workspaces)
            if (kv.first.first == dev && kv.second.ptr)
                if (cudaMemset(kv.second.ptr, 0, 4096) != cudaSuccess) return WQ_ERR_CUDA;
    }
    if (h_fixed != WQ_OK) {
        if (cudaMemset(na->scratch + kNoAllocStatusOffset, 0, sizeof(int)) != cudaSuccess) return WQ_ERR_CUDA;
        if (cudaMemset(na->scratch, 0, 4096) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return h != WQ_OK ? h : h_fixed;
}

namespace {
// The plan of a call on a device with `num_sms` SMs and `smem_optin` bytes of opt-in shared
// memory per block; host arithmetic only.
int fill_plan(int kind, int M, int N, int K, int g, int num_sms, int smem_optin, wq_plan_t* plan) {
    if (!plan) return WQ_ERR_INVALID_ARG;
    int rc = check_shape(K, N);
    if (rc) return rc;
    if (M <= 0) return WQ_ERR_INVALID_ARG;
    if (M > (1 << 24)) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (kind != 0 && kind != 1 && kind != 5 && kind != 6) return WQ_ERR_INVALID_ARG;
    if (num_sms <= 0 || smem_optin <= 0) return WQ_ERR_INVALID_ARG;
    DeviceState d;
    d.num_sms = num_sms;
    d.smem_optin = smem_optin;
    Plan pl;
    rc = plan_for(kind, M, N, K, kind == 1 ? K : g, d, &pl);
    if (rc) return rc;
    plan->grid = pl.grid;
    plan->tile_m = pl.tile_m;
    plan->m_tiles = pl.m_tiles;
    plan->n_tiles = pl.n_tiles;
    plan->k_blocks = pl.k_blocks;
    plan->stages = pl.slots;
    plan->smem_bytes = pl.smem_bytes;
    plan->threads = pl.threads;
    plan->units = pl.units;
    return WQ_OK;
}
}  // namespace

int wq_plan(int kind, int M, int N, int K, int g, wq_plan_t* plan) {
    if (!plan) return WQ_ERR_INVALID_ARG;
    int rc = check_shape(K, N);
    if (rc) return rc;
    if (M <= 0) return WQ_ERR_INVALID_ARG;
    if (kind != 0 && kind != 1 && kind != 5 && kind != 6) return WQ_ERR_INVALID_ARG;
    int num_sms = 0, smem_optin = 0;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int dev = 0;
        DeviceState* d = device_state(&dev);
        if (!d) return WQ_ERR_CUDA;
        if (!d->supported) return WQ_ERR_UNSUPPORTED_DEVICE;
        num_sms = d->num_sms;
        smem_optin = d->smem_optin;
    }
    return fill_plan(kind, M, N, K, g, num_sms, smem_optin, plan);
}

int wq_plan_for(int kind, int M, int N, int K, int g, int num_sms, int smem_optin, wq_plan_t* plan) {
    return fill_plan(kind, M, N, K, g, num_sms, smem_optin, plan);
}

int wq_debug_set_wait_timeout_ns(unsigned long long ns) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_timeout_ns = ns ? ns : kDefaultTimeoutNs;
    return WQ_OK;
}

int wq_debug_skip_publish(int cta) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_skip_publish = cta;
    return WQ_OK;
}

int wq_gemm_w4a16_noalloc(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g,
                          void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = check_shape(K, N);
    if (rc) return rc;
    if (M < 0) return WQ_ERR_INVALID_ARG;
    if (M > (1 << 24)) return WQ_ERR_UNSUPPORTED_SHAPE;
    if (scale_slots(K, g) < 0) return WQ_ERR_INVALID_ARG;
    if (!Wp) return WQ_ERR_INVALID_ARG;
    if (!aligned(Wp, 16)) return WQ_ERR_MISALIGNED;
    if (M == 0) return WQ_OK;
    if (!A || !Y) return WQ_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(Y, 16)) return WQ_ERR_MISALIGNED;

    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    NoAllocDevice* d = nullptr;
    rc = noalloc_device(&dev, &d);
    if (rc) return rc;
    DeviceState ds;
    ds.init = ds.supported = true;
    ds.num_sms = d->num_sms;
    ds.smem_optin = d->smem_optin;
    Plan pl;
    rc = plan_for(0, M, N, K, g, ds, &pl);
    if (rc) return rc;
    if (workspace_bytes_for(pl) > kNoAllocStatusOffset) return WQ_ERR_SCRATCH_LIMIT;
    ActMaps maps;
    rc = encode_activation_maps(&maps, A, M, K, pl.act_rows, pl.chunk, false, !pl.rf);
    if (rc) return rc;
    // the scratch keeps whatever the last call left; the publish flags must start at zero
    if (cudaMemsetAsync(d->scratch, 0, static_cast<size_t>(pl.grid) * sizeof(int), st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }

    // the same launch arguments as wq_gemm_w4a16, with the scratch in place of the workspace
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.wp = static_cast<const uint8_t*>(Wp);
    a.s_chan = (pl.mode == kModeChannel)
                   ? reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(Wp) +
                                                       static_cast<size_t>(pl.n_tiles) * pl.k_blocks * pl.blob_bytes)
                   : nullptr;
    a.y = Y;
    a.ws_flags = reinterpret_cast<int*>(d->scratch);
    a.ws_partial = reinterpret_cast<float*>(d->scratch + 4096);
    a.status = reinterpret_cast<int*>(d->scratch + kNoAllocStatusOffset);
    a.M = M;
    a.N = N;
    a.m_tiles = pl.m_tiles;
    a.n_tiles = pl.n_tiles;
    a.k_blocks = pl.k_blocks;
    a.tile_m = pl.tile_m;
    a.issuers = pl.issuers;
    a.slots = pl.slots;
    a.chunk = pl.chunk;
    a.act_slot = pl.act_slot;
    a.blob_bytes = pl.blob_bytes;
    a.group_rows = g < kTileK ? g : kTileK;
    a.small = pl.small ? 1 : 0;
    a.scale_in_dequant = scale_in_dequant(pl, g);
    a.units = pl.units;
    a.grid = pl.grid;
    a.timeout_ns = g_timeout_ns;
    a.skip_publish = g_skip_publish;
    if (launch_gemm(pl.mode, maps, a, pl, st) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

}  // extern "C"
