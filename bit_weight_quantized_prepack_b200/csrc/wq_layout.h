// Tile geometry and prepacked-weight layout of the library (host and device).
//
// Prepacked W4A16 buffer (the layout pass named by "Efficient Arbitrary Precision
// Acceleration for Large Language Models on GPU Tensor Cores", Abstract: matrix
// preprocessing that reorders data for the kernel; the layout itself is this library's):
//   n-tiles of 128 columns (NT = ceil(N/128)), k-blocks of 128 rows (KT = K/128).
//   Blob (nt, kt) starts at byte (nt*KT + kt) * blob_bytes, so the k-blocks of one column
//   tile are contiguous. A blob is
//     8192 bytes of code words: word ((h*2 + v)*128 + r)*4 + i  (h, v in {0,1}, r < 128,
//       i < 4) holds the 8 codes of column nt*128 + r, rows kt*128 + 64h + 32v + 8i + j
//       (j = 0..7), code j at nibble position kNibblePos[j];
//     then `slots` rows of 128 fp16 scales (slot u covers rows kt*128 + u*min(g,128) ..).
//   For g == K the blobs hold codes only and one row of fp16 column scales (padded to
//   NT*128 entries, then to 16 bytes) follows the last blob.
//   Columns past N hold code 8 and scale 0: zero weights.
// Prepacked W4A8 buffer: the same blobs, codes only, with the W4A8 nibble order.
// Prepacked W4A16 buffer with zero points (g < K): each blob is the W4A16 blob followed by
//   `slots` rows of 128 uint8 zero points z (0..15), laid out like the scale rows; padded
//   columns hold zero point 8 (and scale 0).
// Prepacked 2:4 sparse W4A16 buffer (every run of 4 rows 4i .. 4i+3 of a column holds at most
//   two codes other than 8): the blobs of the W4A16 buffer with the 8192 bytes of code words
//   replaced by 4096 bytes of code words and 2048 bytes of metadata words (then the scale
//   rows, or the column scales after the last blob for g == K). Within blob (nt, kt), 32-row
//   block b < 4 holds pruning groups j < 8 (rows 32b + 4j .. + 3); column c of the tile is in
//   row tile rt = c / 16, with gc = c % 8 and half = (c % 16) / 8:
//     code word (b*8 + rt)*32 + 4gc + (j % 4), nibble half + 2*(j / 4) + 4i: kept code i
//       (0: the lower kept row) of group j of column c;
//     metadata word ((b*8 + rt)*8 + gc)*2 + j / 4, nibble (j % 4) + 4*half: the kept rows'
//       positions in the group, bits 0-1 the lower, bits 2-3 the higher.
//   The kept rows of a group are those whose code is not 8, made up to two with the lowest
//   other rows. Code word 32*(b*8 + rt) + lane is exactly lane's A operand of the sparse warp
//   MMA (m16n8k32, groups of 4 along k) for that row tile and block, and metadata word
//   16*(b*8 + rt) + lane / 2 its metadata operand (lanes 4gc, 4gc + 1).
// Prepacked mixed 2/4-bit W4A16 buffer (a bit width per aligned block of 32 rows x 128
//   columns; a b-bit code q stands for q - 2^(b-1)):
//   a table of NT*KT + 1 uint32 entries (padded to 128 bytes, so that every blob starts on a
//   128-byte boundary): entry nt*KT + kt =
//     (byte offset of blob (nt, kt) / 16) << 4 | wbits (bit v set: 32-row block v is 4-bit),
//     the last entry (end of the blobs / 16) << 4;
//   for g == K, NT*128 fp16 column scales right after the table (padded to 16 bytes);
//   then the blobs, nt-major: for v = 0..3 the block of rows 32v .. 32v + 31, either 2048
//   bytes of 4-bit words laid out as block v of a W4A16 blob (word r*4 + i: rows 32v + 8i +
//   j of column r, nibble kNibblePos[j]) or 1024 bytes of 2-bit words (word rt*32 + 4gc + t:
//   rows 32v + 8t + r of columns 16rt + gc + 8j, 2-bit field r/2 + 4j + 8(r%2)), then the
//   `slots` rows of fp16 scales. Word rt*32 + lane of a 2-bit block is exactly what lane
//   (gc, t) of a warp multiplies for row tile rt: its fields (p, p + 8) are the fp16 pairs of
//   rows 8t + 2s, 8t + 2s + 1 of column 16rt + gc + 8j for p = s + 4j.
//
// Nibble orders. Within a word the W4A16 order puts codes (2p, 2p+1) at nibble positions
// (p, p+4) for p = 0..3, so that masking 0x000F000F (p = 0) or 0x00F000F0 (p = 1) of the
// word, or of the word shifted right by 8 (p = 2, 3), leaves one code in each 16-bit half:
// the two halves become the fp16 pair (k, k+1). The W4A8 order puts codes 0..3 at the low
// nibbles of bytes 0..3 and codes 4..7 at the high nibbles, so that two masks yield four
// int8 lanes in k order each.
#pragma once
#include <cstddef>
#include <cstdint>

namespace wq {

constexpr int kTileN = 128;                   // weight columns per tile = tcgen05 M extent
constexpr int kTileK = 128;                   // weight rows per k-block = one pipeline stage
constexpr int kCodeBytes = kTileN * kTileK / 2;  // 8192 bytes of 4-bit codes per blob
constexpr int kDqResidues = 2;                // large tiles: k-blocks alternate between 2 dequant groups
constexpr int kNumDqWarps = 8 * kDqResidues;  // per group: 4 lane quarters x 2 halves of a k-block
constexpr int kMaxIssuers = 4;                // MMA-issuing warps, one accumulator each
constexpr int kIssuerWarp0 = kNumDqWarps;     // warps 16..19
constexpr int kWeightWarp = kIssuerWarp0 + kMaxIssuers;  // warp 20: weight-blob copies
constexpr int kActWarp = kWeightWarp + 1;     // warp 21: activation-tile copies
constexpr int kThreadsLarge = (kActWarp + 1) * 32;   // 704: epilogue runs in the dequant warps
// small tiles (tile_m <= 32): more warps, each on its own k-blocks
constexpr int kDqWarpsS = 16;                 // 4 per TMEM lane quarter, one per k-block residue (mod 4)
constexpr int kIssuerWarp0S = kDqWarpsS;      // warps 16..19: one MMA issuer per residue
constexpr int kWeightWarpS = kIssuerWarp0S + kMaxIssuers;  // warp 20
constexpr int kActWarpS = kWeightWarpS + 1;   // warp 21
constexpr int kThreadsSmall = (kActWarpS + 1) * 32;  // 704
constexpr int kASlotsS = 4;                   // dequantised k-blocks in tensor memory (small tiles)
constexpr int kSmallTileMax = 32;             // tiles of at most this many rows use per-k-block partials
constexpr int kTmemAOffsetS = 256;            // small tiles: 2 partials per residue in [0, 256), 4 A slots above
constexpr int kMaxTileM = 256;                // activation rows per tile = tcgen05 N extent
// register-operand tiles (M <= kRfMaxM): warp-level MMAs on weights dequantised in registers
constexpr int kRfMaxM = 16;                 // activation rows of two m16n8k16 MMAs
constexpr int kRfWarps = 16;                // 8 column groups of 16 x 2 row halves of 64
constexpr int kWeightWarpR = kRfWarps;      // warp 16
constexpr int kActWarpR = kRfWarps + 1;     // warp 17
constexpr int kThreadsRf = (kActWarpR + 1) * 32;  // 576
constexpr int kMaxSlots = 32;                 // shared-memory ring slots (one k-block each)
constexpr int kMaxChunk = 4;                  // k-blocks moved by one copy
constexpr int kChunkBars = kMaxSlots + 1;     // chunk barriers: more than ring slots
constexpr int kASlots = 4;                    // dequantised weight tiles in tensor memory
constexpr int kTmemCols = 512;
constexpr int kTmemAOffset = 256;             // accumulators in columns [0, 256), A slots above

constexpr int kSpCodeBytes = 4096;           // 2:4 sparse blob: kept codes
constexpr int kSpMetaBytes = 2048;           // then 2-bit positions of the kept codes
constexpr int kSpHeadBytes = kSpCodeBytes + kSpMetaBytes;  // the scale rows start here
constexpr int kSpMinActRows = 8;             // sparse: activation rows per slot (one 128-byte swizzle atom)

constexpr int kMixBlockRows = 32;            // mixed 2/4-bit: rows per width block
constexpr int kMixBlock2 = 1024;             // bytes of a 2-bit block (128 columns x 32 rows)
constexpr int kMixBlock4 = 2048;             // bytes of a 4-bit block

enum Mode : int { kModeGroup = 0, kModeChannel = 1, kModeW4A8 = 2, kModeGroupZP = 3 };

// Scale rows per blob for W4A16; 0 means per-column scales (g == K); -1 unsupported.
inline int scale_slots(int K, int g) {
    if (g <= 0 || K <= 0 || K % g) return -1;
    if (g == K) return 0;
    if (g == 32 || g == 64 || g == 128) return kTileK / g;
    if (g % kTileK == 0) return 1;
    return -1;
}

inline bool shape_ok(int K, int N) { return K > 0 && K % kTileK == 0 && N > 0 && N % 8 == 0; }

inline int n_tiles(int N) { return (N + kTileN - 1) / kTileN; }

inline size_t blob_bytes_w4a16(int slots) { return kCodeBytes + 2u * kTileN * static_cast<size_t>(slots); }

// Asymmetric groups: the W4A16 blob followed by `slots` rows of 128 uint8 zero points.
inline size_t blob_bytes_w4a16_zp(int slots) { return blob_bytes_w4a16(slots) + static_cast<size_t>(kTileN) * slots; }

// 2:4 sparse W4A16: code and metadata words, then `slots` rows of 128 fp16 scales.
inline size_t blob_bytes_sp24(int slots) { return kSpHeadBytes + 2u * kTileN * static_cast<size_t>(slots); }

// Mixed 2/4-bit: bytes of the blob table (NT*KT + 1 uint32 entries, padded to 128 bytes).
inline size_t mixed_table_bytes(long long nblob) { return (static_cast<size_t>(nblob + 1) * 4 + 127) / 128 * 128; }

inline size_t channel_tail_bytes(int N) { return ((2u * n_tiles(N) * kTileN) + 15u) / 16u * 16u; }

}  // namespace wq
