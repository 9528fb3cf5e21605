// damp_internal.h -- host/device shared definitions of libdamp (not installed).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace damp {

// Header written at the start of the caller's pool buffer:
//   [0, 16)                      device status word (uint32) + padding
//   [16, 16 + 16*H)              per-head FP16-row masks, 4 x uint32 (key rows 0..127)
//   [dir_off, dir_off + 528*H)   per-head row directory, 128 x uint32 (see below),
//                                then the head's row-group order (16 bytes)
//   [head_off, head_off + 16*H)  per-head block table, uint4 {block offset inside
//                                the slot, block stride, FP16-row offset, INT8-row
//                                offset} (heads may hold different FP16-row counts)
// rounded up to 256 bytes; the blocks follow, slot s at header + s*slot_stride,
// head h of it at + table[h].x.
//
// Row directory entry of key row i of a quantized block:
//   bits  0..15  byte offset of the row inside the block
//   bits 16..30  byte offset of the row's FP32 scale (INT8 rows; 0 for FP16 rows)
//   bit  31      1 = FP16 row, 0 = INT8 row
//
// Row-group order (read by the d = 128 decode kernel): byte k is the group g
// of key rows [8g, 8g + 8) that half-warp k takes.  Half-warps 2w and 2w + 1
// share warp w, and its format branches diverge on every row position where
// their two groups differ in format; the order pairs the groups so that the
// pairs differ in as few positions as possible (row_group_order).
constexpr size_t kStatusBytes = 16;
constexpr int kMaskWords = 4;
constexpr int kMaxD = 128;
constexpr int kDirWords = 128;               // directory entries per head
constexpr int kDirStride = kDirWords + 4;    // words per head: entries + row-group order
inline size_t dir_offset(int H) { return (kStatusBytes + (size_t)H * kMaskWords * 4 + 15) / 16 * 16; }
inline size_t head_table_offset(int H) { return dir_offset(H) + (size_t)H * kDirStride * 4; }

// Row-group order of a head from its FP16-row mask (4 words, key rows 0..127).
void row_group_order(const uint32_t* mask, uint8_t order[16]);

struct PoolDesc {
    int format;      // DAMP_FMT_*
    int n_slots, H, d;
    int hp;                    // FP16 rows per head; -1 when heads differ
    size_t block_bytes;        // largest algorithmic block size over the heads
    size_t block_stride;       // largest block stride over the heads (stage size)
    size_t slot_stride;        // bytes of one slot (all its heads)
    size_t header_bytes, pool_bytes;
    uint8_t* dev_buf;          // caller's buffer (NULL: host-only descriptor)
    uint32_t* host_masks;      // [H][kMaskWords]
    uint32_t* host_heads;      // [H][4], as the header's block table
    size_t dir_off;            // byte offset of the row directory in the header
    size_t head_off;           // byte offset of the block table in the header
};

// Arguments of the decode-step kernel.
struct StepArgs {
    uint8_t* blocks;           // first block
    const uint32_t* masks;     // [H][4]
    const uint32_t* dir;       // [H][128] row directory
    uint32_t* status;
    const int32_t* slot_idx;
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    float* out;
    const uint4* heads;        // [H] block table (see the header layout)
    unsigned long long slot_stride;
    int n, H, n_slots;
    uint32_t block_stride;     // largest block stride (stage buffer size)
    int n_items;               // work items (groups of 128/d units)
    int n_stages;
    // offsets inside one pipeline stage (bytes)
    uint32_t stage_bytes, st_q, st_k, st_v, st_alpha, st_mask, st_dir, st_meta;
    uint32_t scratch_off;      // start of the consumers' reduction scratch
    uint32_t bar_off;          // start of the mbarriers
};

// Arguments of the pack / unpack kernels.
struct CodecArgs {
    uint8_t* blocks;
    const uint32_t* masks;
    const uint32_t* dir;       // [H][128] row directory (quantized formats)
    uint32_t* status;
    const int32_t* slot_idx;
    float* state;              // [n][H][d][d]
    const uint4* heads;        // [H] block table
    unsigned long long slot_stride;
    int n, H, n_slots;
    int n_items;
};

// Arguments of the calibration accumulate kernel (damp_calib.cu).
struct CalibArgs {
    const float* state;        // first FP32 block of the pool
    uint32_t* status;
    const int32_t* slot_idx;
    const float* alpha;
    double* acc;               // energy [H][d], retention [H][d], count [H]
    int n, H, n_slots, gate;
};

// Launchers (damp_decode.cu, damp_codec.cu, damp_calib.cu).  They return cudaError_t.
cudaError_t launch_decode_step(const PoolDesc& p, const StepArgs& a, int in_dtype, int gate,
                               cudaStream_t stream);
// d = 128 quantized states, one unit per CTA iteration, two CTAs per SM
// (damp_decode_unit.cu); a.n_items counts units (n x H).
cudaError_t launch_decode_unit(const StepArgs& a, int in_dtype, int gate, bool fp8,
                               cudaStream_t stream);
bool decode_unit_fits(const StepArgs& a, int in_dtype, int gate);   // >= 3 stages fit
// One-time kernel attribute set-up for every decode variant a pool can launch
// (called by damp_pool_create, outside any stream capture).
cudaError_t prepare_decode(const PoolDesc& p);
cudaError_t prepare_decode_unit();
cudaError_t launch_calib_accumulate(const CalibArgs& a, int d, cudaStream_t stream);
cudaError_t launch_calib_select(const double* acc, int H, int d, int hp, double* score,
                                uint16_t* idx, cudaStream_t stream);
cudaError_t launch_calib_select_budget(const double* acc, int H, int d, int budget,
                                       double* score, uint8_t* is_fp16, int32_t* hp,
                                       cudaStream_t stream);
cudaError_t launch_pack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream);
cudaError_t launch_unpack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream);

}  // namespace damp
