/*
 * wq.h -- C ABI of the 4-bit weight-quantised linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes Y[M,N] = A[M,K] . W[K,N], with W[k,n] = (q[k,n] - 8) * s[k/g, n]:
 *   - "MARLIN: Mixed-Precision Auto-Regressive Parallel Inference on Large Language Models",
 *     Abstract: a linear layer with weights quantised to 4 bits per element and fp16
 *     activations, kept memory-bound over batch sizes 1..128 by asynchronous memory access,
 *     task scheduling, pipelining and bespoke quantisation support;
 *   - "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method:
 *     fine-grained group quantisation (one scale per group of g rows and column) and
 *     per-token dynamic activation scales;
 *   - "A Speed Odyssey for Deployable Quantization of LLMs", Abstract: the W4A8 kernel
 *     (int8 activations x 4-bit weights), exposed here as wq_gemm_w4a8;
 *   - "Efficient Arbitrary Precision Acceleration for Large Language Models on GPU Tensor
 *     Cores", Abstract: a matrix preprocessing step that reorders the weights into the
 *     layout the kernel reads, exposed here as wq_prepack / wq_prepack_w4a8.
 *
 * Conventions shared by every entry point
 *   - Matrices are dense and row-major. fp16 values are passed as their IEEE binary16 bit
 *     patterns (uint16_t).
 *   - Q holds the 4-bit codes packed 8 per int32 along K: Q is [K/8, N] and code
 *     q[8i+j, n] sits in bits 4j..4j+3 of Q[i, n] (lowest nibble first).
 *   - Every tensor pointer is a DEVICE pointer on the current CUDA device, owned by the
 *     caller; the library never frees or retains it beyond the call's stream work.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls are stream-ordered and asynchronous: they enqueue work and return without
 *     waiting for the device.
 *   - Shapes: K a positive multiple of 128, N a positive multiple of 8, 0 <= M <= 2^24.
 *     M == 0 returns WQ_OK and launches nothing. Group size g: 32, 64, 128, any multiple
 *     of 128 that divides K, or g == K (one scale per column).
 *   - Alignment: A, Q, s, Wp, Y, acc_out: 16 bytes; sa, sw: 4 bytes.
 *   - All preconditions are checked on the host before any launch; a failed check
 *     returns an error status and launches nothing. Launch failures return WQ_ERR_CUDA.
 *     Device-side waits are time-bounded; a wait that expires records WQ_ERR_TIMEOUT in a
 *     per-device status word that wq_get_device_status reports. No call traps or aborts.
 *   - Entry points are thread-safe. Calls in flight at the same time on DIFFERENT streams
 *     use different library workspaces and do not interfere.
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WQ_API __attribute__((visibility("default")))
#else
#define WQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad group size */
    WQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K not a multiple of 128, N not a multiple of 8, M too large */
    WQ_ERR_MISALIGNED = 3,         /* a pointer breaks the alignment rule above */
    WQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
    WQ_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
    WQ_ERR_TIMEOUT = 6,            /* a device-side bounded wait expired (see wq_get_device_status) */
    WQ_ERR_NO_MEMORY = 7,          /* the library could not allocate its workspace */
    WQ_ERR_CAPTURING = 8,          /* the workspace must grow while the stream is being captured */
    WQ_ERR_SCRATCH_LIMIT = 9,      /* wq_gemm_w4a16_noalloc: the plan needs more than its fixed scratch */
    WQ_ERR_NOT_SPARSE = 10         /* wq_prepack_sparse24: the codes are not 2:4 sparse */
} wq_status_t;

/* Human-readable name of a status code. Never NULL. */
WQ_API const char* wq_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
WQ_API int wq_version(void);

/* ---------------------------------------------------------------- prepack (the layout pass)
 * Size in bytes of the prepacked W4A16 buffer for a K x N weight with group size g, or 0
 * when (K, N, g) is not supported. Layout: blobs of 128 columns x 128 rows, each 8192
 * bytes of reordered codes followed by that blob's fp16 group scales; for g == K a single
 * row of fp16 column scales follows all blobs instead. */
WQ_API size_t wq_prepacked_bytes(int K, int N, int g);

/* Size in bytes of the prepacked W4A8 buffer (codes only), or 0 when unsupported. */
WQ_API size_t wq_prepacked_bytes_w4a8(int K, int N);

/* Reorder codes Q [K/8, N] int32 and fp16 scales s [K/g, N] into Wp (caller-allocated,
 * wq_prepacked_bytes(K,N,g) bytes). Columns padded up to a multiple of 128 get code 8 and
 * scale 0, i.e. zero weights. Runs once per weight; Wp is read-only afterwards. */
WQ_API int wq_prepack(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, void* stream);

/* Reorder codes Q [K/8, N] into the W4A8 layout Wp (wq_prepacked_bytes_w4a8 bytes). */
WQ_API int wq_prepack_w4a8(const int32_t* Q, int K, int N, void* Wp, void* stream);

/* Inverse of wq_prepack: recovers Q [K/8, N] and s [K/g, N] bit for bit (test aid). */
WQ_API int wq_unpack(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, void* stream);

/* Inverse of wq_prepack_w4a8 (test aid). */
WQ_API int wq_unpack_w4a8(const void* Wp, int K, int N, int32_t* Q_out, void* stream);

/* ---------------------------------------------------------------- the layer
 * W4A16: Y[M,N] (fp16) = A[M,K] (fp16) . W, W from the prepacked Wp of the same (K, N, g).
 * Products accumulate in fp32; Y is rounded to nearest-even fp16. For g < K the weight
 * (q-8)*s is rounded once to fp16 before the product; for g == K the column scale is
 * applied to the fp32 sum instead. Uses the workspace of (current device, stream).
 * Results are deterministic: the same call gives the same bits every time.
 * The GEMM kernels use programmatic dependent launch: a GEMM may be scheduled while the
 * previous kernel of the stream is still running, but it uses no caller memory (A, Wp, Y,
 * acc_out, sa, sw) until that kernel has completed (before then it only asks L2 to prefetch
 * part of Wp, which reads nothing into the kernel); and it lets the next kernel
 * of the stream start early only if that kernel was itself launched with programmatic
 * stream serialisation (a plain launch still waits for the GEMM to complete). */
WQ_API int wq_gemm_w4a16(const uint16_t* A, const void* Wp, uint16_t* Y,
                  int M, int N, int K, int g, void* stream);

/* ---------------------------------------------------------------- asymmetric groups
 * The layer with a zero point per group and column: W[k,n] = (q[k,n] - z[k/g, n]) * s[k/g, n]
 * ("Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method: fine-grained
 * group quantisation, read with the GPTQ-style 4-bit zero point that the pages leave open;
 * z = 8 everywhere is the symmetric layer). z is uint8 [K/g, N] with values 0..15, 16-byte
 * aligned (a value above 15 is stored as given and gives wrong weights, never an access out
 * of bounds); g must be below K (32, 64, 128 or a multiple of 128 dividing K).
 * wq_prepacked_bytes_zp: the size of the prepacked buffer, or 0 when unsupported; each blob
 * is the W4A16 blob followed by its groups' uint8 zero points (columns padded with z = 8 and
 * s = 0). wq_prepack_zp / wq_unpack_zp: the layout pass and its inverse (test aid), as
 * wq_prepack / wq_unpack. wq_gemm_w4a16_zp: as wq_gemm_w4a16, on the zero-point buffer; the
 * weight (q - z) * s is exact before its one fp16 rounding (none for group scales of
 * g >= 128 on M <= 32, where the scale multiplies each k-block's fp32 partial). */
WQ_API size_t wq_prepacked_bytes_zp(int K, int N, int g);
WQ_API int wq_prepack_zp(const int32_t* Q, const uint16_t* s, const uint8_t* z, int K, int N, int g, void* Wp,
                 void* stream);
WQ_API int wq_unpack_zp(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, uint8_t* z_out,
                 void* stream);
WQ_API int wq_gemm_w4a16_zp(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g,
                 void* stream);

/* ---------------------------------------------------------------- act order
 * Groups whose rows are scattered along K: row k belongs to group g_idx[k] (GPTQ-style
 * act-order checkpoints; "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 * method: one scale, and zero point, per fine-grained group, read with the rows of a group
 * placed anywhere). With perm int32 [K] a permutation of 0..K-1 such that
 * g_idx[perm[i]] == i / g (every group holds exactly g rows; the rows sorted by group, e.g. a
 * stable argsort of g_idx), y = sum_i A[m, perm[i]] * W[perm[i], n] is the grouped layer on the
 * reordered weight and the gathered activations.
 * wq_prepack_act_order: Q int32 [K/8, N] in the checkpoint's row order, s fp16 [K/g, N] and
 * z uint8 [K/g, N] (nullable: the fixed zero point 8) indexed by group -> Wp of
 * wq_prepacked_bytes(K, N, g) bytes (z NULL) or wq_prepacked_bytes_zp(K, N, g) bytes. perm is
 * copied to the host and checked to be a permutation (WQ_ERR_INVALID_ARG otherwise); the call
 * synchronises `stream` and allocates a K/2 * N byte temporary with cudaMallocAsync
 * (WQ_ERR_NO_MEMORY when that fails). Run once per weight.
 * wq_permute_act: A_out fp16 [M, K] = A[:, perm], caller-owned, 16-byte aligned like A and perm;
 * K a positive multiple of 8. An entry of perm outside [0, K) is never dereferenced: its
 * element becomes 0 and the device status word records WQ_ERR_INVALID_ARG
 * (wq_get_device_status reports and clears it).
 * wq_gemm_w4a16_act_order: wq_permute_act into the stream's workspace, then wq_gemm_w4a16
 * (zero_points 0) or wq_gemm_w4a16_zp (zero_points 1) on the act-order buffer, in one call (two
 * launches; the layer's kernel sets up while the gather finishes). The workspace must hold
 * wq_workspace_bytes(4, M, N, K) before the call is captured in a CUDA graph. */
WQ_API int wq_prepack_act_order(const int32_t* Q, const uint16_t* s, const uint8_t* z, const int32_t* perm,
                 int K, int N, int g, void* Wp, void* stream);
WQ_API int wq_permute_act(const uint16_t* A, const int32_t* perm, int M, int K, uint16_t* A_out, void* stream);
WQ_API int wq_gemm_w4a16_act_order(const uint16_t* A, const int32_t* perm, const void* Wp, uint16_t* Y,
                 int M, int N, int K, int g, int zero_points, void* stream);

/* ---------------------------------------------------------------- 2:4 sparse weights
 * The W4A16 layer on a weight in which every run of 4 rows 4i .. 4i+3 of a column holds at
 * most 2 codes other than 8 (2 of every 4 weights are zero): "MARLIN: Mixed-Precision
 * Auto-Regressive Parallel Inference on Large Language Models", Abstract, names the kernel's
 * extension to NVIDIA 2:4 sparsity and gives no format; the one here is this library's own.
 * The buffer keeps the two kept codes of each run and their 2-bit positions: 3/4 of the
 * dense buffer's code bytes. The result is the W4A16 layer of the same (pruned) weight.
 * wq_prepacked_bytes_sparse24: size of the buffer, or 0 when the shape or g is unsupported
 * (g as for wq_gemm_w4a16, g == K included).
 * wq_prepack_sparse24: Q int32 [K/8, N] (pruned codes), s fp16 [K/g, N] -> Wp. Checks the
 * pattern on the device and returns WQ_ERR_NOT_SPARSE when a run holds more than 2 codes
 * other than 8 (Wp's content is then unspecified); the call therefore synchronises `stream`
 * and returns WQ_ERR_CAPTURING while the stream is being captured. Run once per weight.
 * wq_unpack_sparse24: the inverse (test aid): Q_out with the pruned codes as 8, s_out.
 * wq_gemm_w4a16_sparse24: Y [M, N] = A . W as wq_gemm_w4a16 (same rounding: for g = 32 the
 * fp16 weight is rounded once; for g >= 64 the scale multiplies each group's fp32 sum), for
 * 0 <= M <= 16 (WQ_ERR_UNSUPPORTED_SHAPE above: the sparse warp MMA serves the decode-sized
 * batches, where the weight bytes bound the layer). Workspace: wq_workspace_bytes(5, ...). */
WQ_API size_t wq_prepacked_bytes_sparse24(int K, int N, int g);
WQ_API int wq_prepack_sparse24(const int32_t* Q, const uint16_t* s, int K, int N, int g, void* Wp, void* stream);
WQ_API int wq_unpack_sparse24(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, void* stream);
WQ_API int wq_gemm_w4a16_sparse24(const uint16_t* A, const void* Wp, uint16_t* Y, int M, int N, int K, int g,
                 void* stream);

/* ---------------------------------------------------------------- mixed 2/4-bit weights
 * "Enabling Fast 2-bit LLM on GPUs: Memory Alignment and Asynchronous Dequantization",
 * Abstract: most groups of weights at 2 bits, the few groups with a large range at 4 bits,
 * placed with the GPU's memory alignment in mind. Here the width is chosen per aligned block of
 * 32 rows and 128 columns: widths uint8 [K/32, ceil(N/128)] (device memory), each 2 or 4; a
 * b-bit code q stands for q - 2^(b-1), W[k,n] = (q[k,n] - z) * s[k/g, n] with z = 2 or 8 (the
 * block's midpoint). Q keeps the usual 4-bit packing (int32 [K/8, N]); codes of 2-bit blocks
 * must be 0..3. g as for wq_gemm_w4a16, g == K included.
 * wq_prepacked_bytes_mixed: the buffer's size for n4 blocks of 4 bits (0 when unsupported).
 * wq_prepack_mixed: Q, s, widths -> Wp (wp_bytes: the size of the caller's buffer). The call
 * reads the widths on the host (it synchronises `stream`, returns WQ_ERR_CAPTURING while the
 * stream is being captured), writes a blob table (each blob's offset and widths) at the start
 * of Wp, then the blobs of 2-bit (1024 bytes) and 4-bit (2048 bytes) blocks and their scales.
 * WQ_ERR_INVALID_ARG: a width other than 2 or 4, wp_bytes too small, or a code above 3 in a
 * 2-bit block (checked on the device; Wp's content is then unspecified).
 * wq_unpack_mixed: the inverse (test aid): Q_out, s_out and widths_out. It reads the blobs where
 * the buffer's table points, unchecked: pass only a buffer written by wq_prepack_mixed (the
 * layer itself, wq_gemm_w4a16_mixed, checks every blob against wp_bytes before reading it).
 * wq_gemm_w4a16_mixed: Y [M, N] = A . W with the rounding of wq_gemm_w4a16, 0 <= M <= 16
 * (WQ_ERR_UNSUPPORTED_SHAPE above); wp_bytes: the size of the buffer Wp points to (at least
 * wq_prepacked_bytes_mixed(K, N, g, 0), else WQ_ERR_INVALID_ARG). The kernel copies each blob
 * at the offset the table gives only when the blob lies inside wp_bytes and has the size its
 * widths imply; otherwise it copies nothing more, records WQ_ERR_INVALID_ARG in the device
 * status word (wq_get_device_status) and Y is undefined; the call may then last up to the
 * device-side wait limit. Workspace: wq_workspace_bytes(6, ...). */
WQ_API size_t wq_prepacked_bytes_mixed(int K, int N, int g, long long n4);
WQ_API int wq_prepack_mixed(const int32_t* Q, const uint16_t* s, const uint8_t* widths, int K, int N, int g,
                 void* Wp, size_t wp_bytes, void* stream);
WQ_API int wq_unpack_mixed(const void* Wp, int K, int N, int g, int32_t* Q_out, uint16_t* s_out, uint8_t* widths_out,
                 void* stream);
WQ_API int wq_gemm_w4a16_mixed(const uint16_t* A, const void* Wp, size_t wp_bytes, uint16_t* Y, int M, int N,
                 int K, int g, void* stream);

/* W4A8: acc[m,n] = sum_k A[m,k] * (q[k,n] - 8) exactly in int32 (A int8 [M,K]),
 * Y[m,n] = fp16_rn((float(acc) * sa[m]) * sw[n]) with sa fp32 [M] per token and sw fp32
 * [N] per column. acc_out (int32 [M,N]) may be NULL; when given it receives acc.
 * A may hold any int8 value, -128 included. Requires K <= 130944 (the largest multiple of
 * 128 with K * 16384 < 2^31): the kernel sums a * 16(q - 8), whose magnitude reaches
 * 128 * 128 = 16384, in int32, so no partial sum can overflow. */
WQ_API int wq_gemm_w4a8(const int8_t* A, const float* sa, const void* Wp, const float* sw,
                 uint16_t* Y, int32_t* acc_out, int M, int N, int K, void* stream);

/* Per-token activation quantisation, the step before the layer on int8 tensor cores ("Atom:
 * Low-bit Quantization for Efficient and Accurate LLM Serving", method: quantisation
 * parameters of the activations computed from them at inference time, one scale per token;
 * 8-bit activations for W4A8, 4-bit for W4A4). With L = 127 (bits = 8) or 7 (bits = 4), for
 * each row m of the fp16 activations A [M, K]: amax = max_k |A[m,k]|, inv = L / amax and
 * sa[m] = amax / L (fp32 divisions, round to nearest), A_q[m,k] = round-half-even(A[m,k] *
 * inv) (fp32 product, round to nearest) clamped to [-L, L]; a row of zeros gives codes 0 and
 * sa[m] = 0. 4-bit codes are stored one per int8 (unpacked: tcgen05 has no 4-bit integer
 * MMA). A must be finite. A_q int8 [M, K] and sa fp32 [M] are caller-owned device memory.
 * K a positive multiple of 8, 0 <= M <= 2^24; A and A_q 16-byte aligned, sa 4-byte. */
WQ_API int wq_quantize_act(const uint16_t* A, int M, int K, int bits, int8_t* A_q, float* sa, void* stream);

/* The layer on fp16 activations quantised per token to act_bits = 8 (W4A8) or 4 (W4A4):
 * wq_quantize_act into the stream's workspace, then wq_gemm_w4a8 on the codes and scales, in
 * one call (two launches on `stream`; the layer's kernel sets up and prefetches its first
 * weight blobs while the quantisation finishes, and reads the codes only after it). Y,
 * acc_out and the constraints are those of wq_gemm_w4a8; sa_out (fp32 [M], nullable)
 * receives the per-token scales. The workspace must hold wq_workspace_bytes(2, M, N, K)
 * bytes (it grows on first use, or by wq_workspace_reserve). */
WQ_API int wq_gemm_w4a8_fp16act(const uint16_t* A, const void* Wp, const float* sw, uint16_t* Y,
                 int32_t* acc_out, float* sa_out, int M, int N, int K, int act_bits, void* stream);

/* W4A16 without any allocation. No counterpart in the paper: it exists for callers that
 * cannot allocate device memory when they run the layer (an engine that gave all free
 * memory to its own pool at start-up, a plugin whose host framework owns every
 * allocation, a latency-critical loop that must not risk an allocation's implicit
 * synchronisation). Same arguments and result bits as wq_gemm_w4a16, but
 * the stream-K scratch (publish flags, partial tiles) lives in one fixed array of
 * WQ_NOALLOC_SCRATCH_BYTES (8 MiB) that every device loading the library holds until
 * the process exits; this call never calls cudaMalloc or cudaFree.
 * - Limit: a plan whose scratch (4 KiB + grid * tile rows * 128 * 4 bytes) does not fit
 *   returns WQ_ERR_SCRATCH_LIMIT and launches nothing. On a 148-SM B200 every M <= 64
 *   fits; larger M (tiles of 128 or 256 rows) does not.
 * - Set-up: the first call on a device (with that device current) configures the
 *   kernels, looks up the array's device address and clears it with blocking memsets;
 *   make that first call before any stream capture.
 * - Every call clears the publish flags on `stream` before its kernel, so a call does not
 *   depend on what an earlier one left in the array.
 * - All calls on one device share the array: two calls whose kernels overlap on the GPU
 *   (different streams without ordering between them) race and give wrong results.
 *   Order them on one stream or with events.
 * - A device-side wait that expires stops the kernel as in wq_gemm_w4a16; it is recorded in
 *   the array's own status word, which wq_get_device_status reads and clears as well
 *   (without allocating). */
#define WQ_NOALLOC_SCRATCH_BYTES (8u << 20)
WQ_API int wq_gemm_w4a16_noalloc(const uint16_t* A, const void* Wp, uint16_t* Y,
                  int M, int N, int K, int g, void* stream);

/* ---------------------------------------------------------------- workspace and status
 * Bytes of library workspace one call of the given kind and shape needs (kind 0 = W4A16,
 * 1 = W4A8, 2 = W4A8 on fp16 activations, wq_gemm_w4a8_fp16act, 3 = wq_gemm_w4a16_zp,
 * 4 = wq_gemm_w4a16_act_order, 5 = wq_gemm_w4a16_sparse24, 6 = wq_gemm_w4a16_mixed (0 for
 * M > 16 for the last two)). */
WQ_API size_t wq_workspace_bytes(int kind, int M, int N, int K);

/* Make sure the workspace of (current device, stream) holds at least `bytes`. Call it
 * before capturing the stream into a CUDA graph: a call that has to grow the workspace
 * while the stream is capturing returns WQ_ERR_CAPTURING. Synchronises `stream` when it
 * grows the buffer. A workspace (one int32 flag and one tile_m x 128 fp32 partial per CTA,
 * at least 1 MiB) is kept for the life of the process; each stream used gets its own, so
 * calls on different streams may overlap. */
WQ_API int wq_workspace_reserve(size_t bytes, void* stream);

/* Synchronise `stream`, then return and clear the current device's status words (that of
 * the workspace calls and that of wq_gemm_w4a16_noalloc): WQ_OK, or WQ_ERR_TIMEOUT when a
 * device-side wait expired since the last call. The outputs of the call whose wait expired
 * are undefined, and so are those of every later call on the same stream (or, for
 * wq_gemm_w4a16_noalloc, on the same device) until this function has returned: an expired
 * wait can leave stream-K flags set, and only this function clears them. */
WQ_API int wq_get_device_status(void* stream);

/* ---------------------------------------------------------------- introspection and test hooks
 * The launch plan a call would use. kind 0 = W4A16, 1 = W4A8, 5 = 2:4 sparse W4A16, 6 = mixed
 * 2/4-bit W4A16 (5 and 6: M <= 16). */
typedef struct {
    int grid;         /* persistent CTAs launched (<= number of SMs) */
    int tile_m;       /* activation rows per tile: 1, 2, 4, 8 or 16 for the register-operand kernel
                         (M <= 16), else the tcgen05 MMA's N extent (32..256) */
    int m_tiles;      /* tiles along M */
    int n_tiles;      /* tiles of 128 columns along N */
    int k_blocks;     /* blocks of 128 rows along K */
    int stages;       /* shared-memory pipeline depth */
    int smem_bytes;   /* dynamic shared memory per CTA */
    int threads;      /* threads per CTA: 576 for the register-operand kernel, 704 otherwise */
    long long units;  /* (tile, k-block) work units split across the CTAs */
} wq_plan_t;
WQ_API int wq_plan(int kind, int M, int N, int K, int g, wq_plan_t* plan);

/* The same plan for a device with `num_sms` SMs and `smem_optin` bytes of opt-in dynamic
 * shared memory per block, without touching any device (host arithmetic only; usable on a
 * machine without a GPU). Arguments are checked as for wq_plan; num_sms and smem_optin must
 * be positive; WQ_ERR_UNSUPPORTED_SHAPE when no pipeline of two stages fits. */
WQ_API int wq_plan_for(int kind, int M, int N, int K, int g, int num_sms, int smem_optin, wq_plan_t* plan);

/* Test hooks. wq_debug_set_wait_timeout_ns sets the limit of every device-side wait
 * (default 2e9 ns; 0 restores the default). wq_debug_skip_publish(c) makes CTA c skip
 * publishing its partial sum to the tile that owns it (c = -1 disables), so that the
 * owner's bounded wait expires: the call then reports WQ_ERR_TIMEOUT through
 * wq_get_device_status instead of hanging. Both apply to later calls on every device, of
 * wq_gemm_w4a16, wq_gemm_w4a8 and wq_gemm_w4a16_noalloc alike. */
WQ_API int wq_debug_set_wait_timeout_ns(unsigned long long ns);
WQ_API int wq_debug_skip_publish(int cta);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
