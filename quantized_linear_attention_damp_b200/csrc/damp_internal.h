// damp_internal.h -- host/device shared definitions of libdamp (not installed).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace damp {

// Header written at the start of the caller's pool buffer:
//   [0, 16)                      device status word (uint32) + padding
//   [16, 16 + 32*H)              per-head FP16-row masks, 8 x uint32 (key rows 0..255)
//   [dir_off, dir_off + 4*d_k*H) per-head row directory, d_k x uint32 (see below)
//   [head_off, head_off + 16*H)  per-head block table, uint4 {block offset inside
//                                the slot, block stride, FP16-row offset, INT8-row
//                                offset} (heads may hold different FP16-row counts)
// rounded up to 256 bytes; the blocks follow, slot s at header + s*slot_stride,
// head h of it at + table[h].x.
//
// Row directory entry of key row i of a quantized block:
//   bits  0..17  byte offset of the row inside the block
//   bits 18..30  index of the row's FP32 scale among the block's scales (byte
//                offset / 4; INT8 and FP8 rows; 0 for FP16 rows)
//   bit  31      1 = FP16 row, 0 = byte row (INT8 or FP8 E4M3)
constexpr size_t kStatusBytes = 16;
constexpr int kMaxDim = 256;                  // largest d_k and d_v
constexpr int kMaskWords = kMaxDim / 32;      // FP16-row mask words per head
constexpr int kMaxFastD = 128;                // largest d of the square fast kernels
__host__ __device__ inline uint32_t dir_row(uint32_t e) { return e & 0x3ffffu; }
__host__ __device__ inline uint32_t dir_scale(uint32_t e) { return (e >> 16) & 0x7ffcu; }
__host__ __device__ inline uint32_t dir_entry(uint32_t row_off, uint32_t scale_off, bool f16) {
    return row_off | ((scale_off >> 2) << 18) | (f16 ? 0x80000000u : 0u);
}
// An FP16 row of d_v values is stored as two planes of d_v bytes: values 4g
// and 4g + 1 of column group g in the first plane at byte 4g, values 4g + 2
// and 4g + 3 in the second at d_v + 4g.  A thread holding the 4 columns of
// group g then reads an FP16 row with the same 4-byte stride as a byte row
// (one word in each plane, the byte row's word at the same offset as the
// first).  Byte offset of value j:
__host__ __device__ inline uint32_t f16_pos(uint32_t j, uint32_t d_v) {
    return ((j >> 1) & 1u) * d_v + 4u * (j >> 2) + 2u * (j & 1u);
}
inline size_t dir_offset(int H) { return (kStatusBytes + (size_t)H * kMaskWords * 4 + 15) / 16 * 16; }
inline size_t head_table_offset(int H, int d_k) { return dir_offset(H) + (size_t)H * d_k * 4; }

struct PoolDesc {
    int format;      // DAMP_FMT_*
    int n_slots, H, d_k, d_v;
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
    const uint32_t* masks;     // [H][kMaskWords]
    const uint32_t* dir;       // [H][d_k] row directory
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
    int d_k, d_v;
    int format;                // DAMP_FMT_*
    uint32_t block_stride;     // largest block stride (stage buffer size)
    int n_items;               // work items (groups of 128/d units)
    int n_stages;
    // offsets inside one pipeline stage (bytes)
    uint32_t stage_bytes, st_q, st_k, st_v, st_alpha, st_mask, st_dir, st_meta;
    uint32_t scratch_off;      // start of the consumers' reduction scratch
    uint32_t bar_off;          // start of the mbarriers
    unsigned long long wait_ns;   // bound of every pipeline wait (ns)
    uint32_t hooks;            // test hooks (kHookHoldFirstItem)
    int validate;              // 1: units with a non-finite input are skipped and flagged
};

// Test hook of the failure path: the refill side of every CTA never issues its
// first item (no copy, no arrival), so the consumers' bounded wait for it runs
// out and the kernel takes its abort path.
constexpr uint32_t kHookHoldFirstItem = 1u;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;   // 2 s

// Arguments of the pack / unpack kernels.
struct CodecArgs {
    uint8_t* blocks;
    const uint32_t* masks;
    const uint32_t* dir;       // [H][d_k] row directory (quantized formats)
    uint32_t* status;
    const int32_t* slot_idx;
    float* state;              // [n][H][d_k][d_v]
    const uint4* heads;        // [H] block table
    unsigned long long slot_stride;
    int n, H, n_slots;
    int d_k, d_v;
    int format;                // DAMP_FMT_*
    int n_items;
};

// Arguments of the calibration accumulate kernel (damp_calib.cu).
struct CalibArgs {
    const float* state;        // first FP32 block of the pool
    uint32_t* status;
    const int32_t* slot_idx;
    const float* alpha;
    double* acc;               // energy [H][d_k], retention [H][d_k], count [H]
    int n, H, n_slots, gate;
    int d_k, d_v;
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
// Any d_k x d_v (multiples of 16 up to 256), every format: one CTA per unit
// (damp_decode_any.cu); used where no fast kernel fits.
cudaError_t launch_decode_any(const StepArgs& a, int in_dtype, int gate, cudaStream_t stream);
cudaError_t launch_pack_any(const CodecArgs& a, cudaStream_t stream);
cudaError_t launch_unpack_any(const CodecArgs& a, cudaStream_t stream);
cudaError_t launch_calib_accumulate(const CalibArgs& a, cudaStream_t stream);
cudaError_t launch_calib_select(const double* acc, int H, int d, int hp, double* score,
                                uint16_t* idx, cudaStream_t stream);
cudaError_t launch_calib_select_budget(const double* acc, int H, int d, int budget,
                                       double* score, uint8_t* is_fp16, int32_t* hp,
                                       cudaStream_t stream);
cudaError_t launch_pack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream);
cudaError_t launch_unpack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream);

}  // namespace damp
