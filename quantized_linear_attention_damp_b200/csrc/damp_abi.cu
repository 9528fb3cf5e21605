// damp_abi.cu -- the C ABI of libdamp (declared in include/damp.h).
//
// Host-side argument checks, the pool descriptor and its header, the block
// layout, and the host-only conversions between raw blocks and the logical
// per-row form.  Every check happens before anything is enqueued; kernels
// report device-side conditions through the pool's status word.
#include <cuda_runtime.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <new>
#include <thread>
#include <vector>

#include "damp.h"
#include "damp_internal.h"

using damp::PoolDesc;

struct damp_pool {
    PoolDesc d;
};


namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dim_ok(int d) { return d >= 16 && d <= damp::kMaxDim && d % 16 == 0; }

int check_shape(int format, int d_k, int d_v, int hp_rows) {
    if (format != DAMP_FMT_FP32 && format != DAMP_FMT_INT8_ROW && format != DAMP_FMT_MIXED &&
        format != DAMP_FMT_FP8_ROW)
        return DAMP_ERR_INVALID_ARGUMENT;
    if (!dim_ok(d_k) || !dim_ok(d_v)) return DAMP_ERR_UNSUPPORTED;
    if (hp_rows < 0 || hp_rows > d_k) return DAMP_ERR_INVALID_ARGUMENT;
    if (format != DAMP_FMT_MIXED && hp_rows != 0) return DAMP_ERR_INVALID_ARGUMENT;
    return DAMP_OK;
}

void layout(int format, int d_k, int d_v, int hp, size_t* bytes, size_t* stride,
            uint32_t* f16_off, uint32_t* i8_off) {
    if (format == DAMP_FMT_FP32) {
        *bytes = (size_t)d_k * d_v * 4;
        *stride = *bytes;
        *f16_off = *i8_off = 0;
        return;
    }
    const size_t r = (size_t)(d_k - hp);
    *bytes = 4 * r + 2 * (size_t)hp * d_v + r * d_v;
    const size_t scales = align_up(4 * r, 16);
    *f16_off = (uint32_t)scales;
    *i8_off = (uint32_t)(scales + 2 * (size_t)hp * d_v);
    *stride = align_up(scales + 2 * (size_t)hp * d_v + r * d_v, 16);
}

size_t header_bytes(int H, int d_k) {
    return align_up(damp::head_table_offset(H, d_k) + (size_t)H * 16, 256);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? DAMP_OK : DAMP_ERR_CUDA; }

bool is_fp16_row(const PoolDesc& d, int h, int i) {
    return (d.host_masks[(size_t)h * damp::kMaskWords + (i >> 5)] >> (i & 31)) & 1u;
}

}  // namespace

extern "C" {

const char* damp_status_string(int status) {
    switch (status) {
        case DAMP_OK: return "ok";
        case DAMP_ERR_INVALID_ARGUMENT: return "invalid argument";
        case DAMP_ERR_UNSUPPORTED:
            return "unsupported shape (d_k, d_v multiples of 16 in [16, 256])";
        case DAMP_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case DAMP_ERR_BUFFER_TOO_SMALL: return "pool buffer too small";
        case DAMP_ERR_CUDA: return "CUDA runtime error";
        case DAMP_ERR_TIMEOUT: return "host wait on the stream timed out";
        default: return "unknown status";
    }
}

int damp_layout(int format, int d_k, int d_v, int hp_rows, size_t* block_bytes,
                size_t* block_stride) {
    const int rc = check_shape(format, d_k, d_v, hp_rows);
    if (rc) return rc;
    size_t b, s;
    uint32_t f, i;
    layout(format, d_k, d_v, hp_rows, &b, &s, &f, &i);
    if (block_bytes) *block_bytes = b;
    if (block_stride) *block_stride = s;
    return DAMP_OK;
}

}  // extern "C"

namespace {

// Per-head layout of a pool whose FP16-row masks are known: the block table
// (offset inside the slot, stride, FP16-row offset, INT8-row offset), the
// slot stride, the largest block size and stride.
struct Layout {
    std::vector<uint32_t> heads;   // [H][4]
    size_t slot_stride = 0, max_bytes = 0, max_stride = 0;
};

Layout pool_layout(int format, int H, int d_k, int d_v, const std::vector<uint32_t>& masks) {
    Layout L;
    L.heads.assign((size_t)H * 4, 0u);
    for (int h = 0; h < H; ++h) {
        int hp = 0;
        for (int w = 0; w < damp::kMaskWords; ++w)
            hp += __builtin_popcount(masks[(size_t)h * damp::kMaskWords + w]);
        size_t b, st;
        uint32_t f16, i8;
        layout(format, d_k, d_v, hp, &b, &st, &f16, &i8);
        uint32_t* e = &L.heads[(size_t)h * 4];
        e[0] = (uint32_t)L.slot_stride;
        e[1] = (uint32_t)st;
        e[2] = f16;
        e[3] = i8;
        L.slot_stride += st;
        if (b > L.max_bytes) L.max_bytes = b;
        if (st > L.max_stride) L.max_stride = st;
    }
    return L;
}

}  // namespace

extern "C" {

int damp_pool_bytes(int format, int n_slots, int H, int d_k, int d_v, int hp_rows,
                    size_t* bytes) {
    if (!bytes || n_slots < 1 || H < 1) return DAMP_ERR_INVALID_ARGUMENT;
    const int rc = check_shape(format, d_k, d_v, hp_rows);
    if (rc) return rc;
    size_t b, s;
    uint32_t f, i;
    layout(format, d_k, d_v, hp_rows, &b, &s, &f, &i);
    *bytes = header_bytes(H, d_k) + (size_t)n_slots * H * s;
    return DAMP_OK;
}

}  // extern "C"

namespace {

// Masks from a per-head FP16-row map (0/1 bytes, [H][d_k]).
int masks_from_map(int H, int d_k, const uint8_t* is_fp16, std::vector<uint32_t>* masks) {
    masks->assign((size_t)H * damp::kMaskWords, 0u);
    for (int h = 0; h < H; ++h)
        for (int i = 0; i < d_k; ++i) {
            const uint8_t f = is_fp16[(size_t)h * d_k + i];
            if (f > 1) return DAMP_ERR_INVALID_ARGUMENT;
            if (f) (*masks)[(size_t)h * damp::kMaskWords + (i >> 5)] |= 1u << (i & 31);
        }
    return DAMP_OK;
}

int create_common(int format, int n_slots, int H, int d_k, int d_v, int hp_rows,
                  const std::vector<uint32_t>& masks, void* dev_buf, size_t buf_bytes,
                  damp_pool** out) {
    const Layout L = pool_layout(format, H, d_k, d_v, masks);
    if (L.slot_stride > 0xffffffffull) return DAMP_ERR_UNSUPPORTED;
    PoolDesc d{};
    d.format = format;
    d.n_slots = n_slots;
    d.H = H;
    d.d_k = d_k;
    d.d_v = d_v;
    d.hp = hp_rows;
    d.block_bytes = L.max_bytes;
    d.block_stride = L.max_stride;
    d.slot_stride = L.slot_stride;
    d.header_bytes = header_bytes(H, d_k);
    d.dir_off = damp::dir_offset(H);
    d.head_off = damp::head_table_offset(H, d_k);
    d.pool_bytes = d.header_bytes + (size_t)n_slots * d.slot_stride;
    if (dev_buf) {
        if (!aligned16(dev_buf)) return DAMP_ERR_MISALIGNED;
        if (buf_bytes < d.pool_bytes) return DAMP_ERR_BUFFER_TOO_SMALL;
    }
    damp_pool* p = new (std::nothrow) damp_pool;
    if (!p) return DAMP_ERR_INVALID_ARGUMENT;
    p->d = d;
    p->d.dev_buf = static_cast<uint8_t*>(dev_buf);
    p->d.host_masks = new (std::nothrow) uint32_t[masks.size()];
    p->d.host_heads = new (std::nothrow) uint32_t[L.heads.size()];
    if (!p->d.host_masks || !p->d.host_heads) {
        delete[] p->d.host_masks;
        delete[] p->d.host_heads;
        delete p;
        return DAMP_ERR_INVALID_ARGUMENT;
    }
    memcpy(p->d.host_masks, masks.data(), masks.size() * 4);
    memcpy(p->d.host_heads, L.heads.data(), L.heads.size() * 4);
    if (dev_buf) {
        std::vector<uint8_t> hdr(d.header_bytes, 0);
        memcpy(hdr.data() + damp::kStatusBytes, masks.data(), masks.size() * 4);
        memcpy(hdr.data() + d.head_off, L.heads.data(), L.heads.size() * 4);
        if (format != DAMP_FMT_FP32) {
            // row directory: offsets of each key row (and its scale) in its head's block
            uint32_t* dir = reinterpret_cast<uint32_t*>(hdr.data() + d.dir_off);
            for (int h = 0; h < H; ++h) {
                const uint32_t f16_off = L.heads[(size_t)h * 4 + 2];
                const uint32_t i8_off = L.heads[(size_t)h * 4 + 3];
                uint32_t r16 = 0, r8 = 0;
                for (int i = 0; i < d_k; ++i) {
                    const bool f16 = (masks[(size_t)h * damp::kMaskWords + (i >> 5)] >> (i & 31)) & 1u;
                    uint32_t e;
                    if (f16) {
                        e = damp::dir_entry(f16_off + r16 * 2u * (uint32_t)d_v, 0u, true);
                        ++r16;
                    } else {
                        e = damp::dir_entry(i8_off + r8 * (uint32_t)d_v, 4u * r8, false);
                        ++r8;
                    }
                    dir[(size_t)h * d_k + i] = e;
                }
            }
        }
        cudaError_t e = cudaMemcpy(dev_buf, hdr.data(), hdr.size(), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = damp::prepare_decode(d);
        if (e != cudaSuccess) {
            delete[] p->d.host_masks;
            delete[] p->d.host_heads;
            delete p;
            return DAMP_ERR_CUDA;
        }
    }
    *out = p;
    return DAMP_OK;
}

}  // namespace

extern "C" {

int damp_pool_create(int format, int n_slots, int H, int d_k, int d_v, int hp_rows,
                     const uint16_t* hp_row_idx, void* dev_buf, size_t buf_bytes,
                     damp_pool** out) {
    if (!out) return DAMP_ERR_INVALID_ARGUMENT;
    *out = nullptr;
    if (n_slots < 1 || H < 1) return DAMP_ERR_INVALID_ARGUMENT;
    int rc = check_shape(format, d_k, d_v, hp_rows);
    if (rc) return rc;
    if (hp_rows > 0 && !hp_row_idx) return DAMP_ERR_INVALID_ARGUMENT;
    std::vector<uint32_t> masks((size_t)H * damp::kMaskWords, 0u);
    for (int h = 0; h < H; ++h)
        for (int j = 0; j < hp_rows; ++j) {
            const int i = hp_row_idx[(size_t)h * hp_rows + j];
            if (i >= d_k) return DAMP_ERR_INVALID_ARGUMENT;
            uint32_t& w = masks[(size_t)h * damp::kMaskWords + (i >> 5)];
            if (w & (1u << (i & 31))) return DAMP_ERR_INVALID_ARGUMENT;  // repeated row
            w |= 1u << (i & 31);
        }
    return create_common(format, n_slots, H, d_k, d_v, hp_rows, masks, dev_buf, buf_bytes, out);
}

int damp_pool_bytes_map(int n_slots, int H, int d_k, int d_v, const uint8_t* is_fp16,
                        size_t* bytes) {
    if (!bytes || !is_fp16 || n_slots < 1 || H < 1) return DAMP_ERR_INVALID_ARGUMENT;
    int rc = check_shape(DAMP_FMT_MIXED, d_k, d_v, 0);
    if (rc) return rc;
    std::vector<uint32_t> masks;
    if ((rc = masks_from_map(H, d_k, is_fp16, &masks))) return rc;
    const Layout L = pool_layout(DAMP_FMT_MIXED, H, d_k, d_v, masks);
    *bytes = header_bytes(H, d_k) + (size_t)n_slots * L.slot_stride;
    return DAMP_OK;
}

int damp_pool_create_map(int n_slots, int H, int d_k, int d_v, const uint8_t* is_fp16,
                         void* dev_buf, size_t buf_bytes, damp_pool** out) {
    if (!out) return DAMP_ERR_INVALID_ARGUMENT;
    *out = nullptr;
    if (n_slots < 1 || H < 1 || !is_fp16) return DAMP_ERR_INVALID_ARGUMENT;
    int rc = check_shape(DAMP_FMT_MIXED, d_k, d_v, 0);
    if (rc) return rc;
    std::vector<uint32_t> masks;
    if ((rc = masks_from_map(H, d_k, is_fp16, &masks))) return rc;
    // one FP16-row count for every head -> the same pool as damp_pool_create
    int hp = -1;
    for (int h = 0; h < H; ++h) {
        int c = 0;
        for (int w = 0; w < damp::kMaskWords; ++w)
            c += __builtin_popcount(masks[(size_t)h * damp::kMaskWords + w]);
        hp = (h == 0 || c == hp) ? c : -2;
    }
    return create_common(DAMP_FMT_MIXED, n_slots, H, d_k, d_v, hp < 0 ? -1 : hp, masks, dev_buf,
                         buf_bytes, out);
}

int damp_pool_head_layout(const damp_pool* pool, int h, size_t* block_bytes,
                          size_t* block_stride, size_t* offset_in_slot) {
    if (!pool || h < 0 || h >= pool->d.H) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    const uint32_t* e = d.host_heads + (size_t)h * 4;
    if (block_bytes) {
        if (d.format == DAMP_FMT_FP32) {
            *block_bytes = (size_t)d.d_k * d.d_v * 4;
        } else {
            const size_t r = (size_t)(e[3] - e[2]) / (2 * (size_t)d.d_v);   // FP16 rows
            const size_t r8 = (size_t)d.d_k - r;
            *block_bytes = 4 * r8 + 2 * r * d.d_v + r8 * d.d_v;
        }
    }
    if (block_stride) *block_stride = e[1];
    if (offset_in_slot) *offset_in_slot = e[0];
    return DAMP_OK;
}

int damp_pool_destroy(damp_pool* pool) {
    if (!pool) return DAMP_OK;
    delete[] pool->d.host_masks;
    delete[] pool->d.host_heads;
    delete pool;
    return DAMP_OK;
}

int damp_pool_block_offset(const damp_pool* pool, int slot, int h, size_t* offset) {
    if (!pool || !offset) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    if (slot < 0 || slot >= d.n_slots || h < 0 || h >= d.H) return DAMP_ERR_INVALID_ARGUMENT;
    *offset = d.header_bytes + (size_t)slot * d.slot_stride + d.host_heads[(size_t)h * 4];
    return DAMP_OK;
}

static int codec_args(const damp_pool* pool, int n, const int32_t* slot_idx, const float* state,
                      damp::CodecArgs* a) {
    if (!pool || n < 0) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    if (!d.dev_buf) return DAMP_ERR_INVALID_ARGUMENT;
    if (n == 0) return 1;  // nothing to do
    if (!slot_idx || !state) return DAMP_ERR_INVALID_ARGUMENT;
    if (!aligned16(state) || (reinterpret_cast<uintptr_t>(slot_idx) & 3u))
        return DAMP_ERR_MISALIGNED;
    a->blocks = d.dev_buf + d.header_bytes;
    a->masks = reinterpret_cast<const uint32_t*>(d.dev_buf + damp::kStatusBytes);
    a->dir = reinterpret_cast<const uint32_t*>(d.dev_buf + d.dir_off);
    a->status = reinterpret_cast<uint32_t*>(d.dev_buf);
    a->slot_idx = slot_idx;
    a->state = const_cast<float*>(state);
    a->n = n;
    a->H = d.H;
    a->n_slots = d.n_slots;
    a->heads = reinterpret_cast<const uint4*>(d.dev_buf + d.head_off);
    a->slot_stride = d.slot_stride;
    a->d_k = d.d_k;
    a->d_v = d.d_v;
    a->format = d.format;
    a->n_items = n * d.H;   // units (the launcher groups them)
    return DAMP_OK;
}

int damp_pool_pack(const damp_pool* pool, int n, const int32_t* slot_idx, const float* state,
                   void* stream) {
    damp::CodecArgs a{};
    const int rc = codec_args(pool, n, slot_idx, state, &a);
    if (rc) return rc < 0 ? rc : DAMP_OK;
    return cuda_status(damp::launch_pack(pool->d, a, static_cast<cudaStream_t>(stream)));
}

int damp_pool_unpack(const damp_pool* pool, int n, const int32_t* slot_idx, float* state,
                     void* stream) {
    damp::CodecArgs a{};
    const int rc = codec_args(pool, n, slot_idx, state, &a);
    if (rc) return rc < 0 ? rc : DAMP_OK;
    return cuda_status(damp::launch_unpack(pool->d, a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Test hooks of the failure path (damp_set_test_hooks).
std::atomic<unsigned long long> g_wait_ns{0};
std::atomic<uint32_t> g_hooks{0};

int decode_common(const damp_pool* pool, int n, const int32_t* slot_idx, int in_dtype,
                  const void* q, const void* k, const void* v, int gate, const float* alpha,
                  const float* beta, float* out, void* stream, int validate) {
    if (!pool || n < 0) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    if (!d.dev_buf) return DAMP_ERR_INVALID_ARGUMENT;
    if (in_dtype != DAMP_DTYPE_BF16 && in_dtype != DAMP_DTYPE_F32) return DAMP_ERR_INVALID_ARGUMENT;
    if (gate != DAMP_GATE_SCALAR && gate != DAMP_GATE_VECTOR) return DAMP_ERR_INVALID_ARGUMENT;
    if (n == 0) return DAMP_OK;
    if (!slot_idx || !q || !k || !v || !alpha || !beta || !out) return DAMP_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return DAMP_ERR_MISALIGNED;
    if (gate == DAMP_GATE_VECTOR && !aligned16(alpha)) return DAMP_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(slot_idx) & 3u) || (reinterpret_cast<uintptr_t>(beta) & 3u) ||
        (reinterpret_cast<uintptr_t>(alpha) & 3u))
        return DAMP_ERR_MISALIGNED;
    if ((size_t)n * d.H > (size_t)0x7fffffff) return DAMP_ERR_UNSUPPORTED;
    damp::StepArgs a{};
    a.d_k = d.d_k;
    a.d_v = d.d_v;
    a.format = d.format;
    a.blocks = d.dev_buf + d.header_bytes;
    a.masks = reinterpret_cast<const uint32_t*>(d.dev_buf + damp::kStatusBytes);
    a.dir = reinterpret_cast<const uint32_t*>(d.dev_buf + d.dir_off);
    a.status = reinterpret_cast<uint32_t*>(d.dev_buf);
    a.slot_idx = slot_idx;
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.out = out;
    a.n = n;
    a.H = d.H;
    a.n_slots = d.n_slots;
    a.heads = reinterpret_cast<const uint4*>(d.dev_buf + d.head_off);
    a.slot_stride = d.slot_stride;
    a.block_stride = (uint32_t)d.block_stride;
    a.n_items = n * d.H;   // units (the launcher groups them)
    const unsigned long long wait = g_wait_ns.load(std::memory_order_relaxed);
    a.wait_ns = wait ? wait : damp::kDefaultWaitNs;
    a.hooks = g_hooks.load(std::memory_order_relaxed);
    a.validate = validate;
    return cuda_status(
        damp::launch_decode_step(d, a, in_dtype, gate, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int damp_decode_step(const damp_pool* pool, int n, const int32_t* slot_idx, int in_dtype,
                     const void* q, const void* k, const void* v, int gate, const float* alpha,
                     const float* beta, float* out, void* stream) {
    return decode_common(pool, n, slot_idx, in_dtype, q, k, v, gate, alpha, beta, out, stream, 0);
}

int damp_decode_step_validated(const damp_pool* pool, int n, const int32_t* slot_idx,
                               int in_dtype, const void* q, const void* k, const void* v,
                               int gate, const float* alpha, const float* beta, float* out,
                               void* stream) {
    return decode_common(pool, n, slot_idx, in_dtype, q, k, v, gate, alpha, beta, out, stream, 1);
}

int damp_set_test_hooks(uint64_t wait_limit_ns, uint32_t hooks) {
    if (hooks & ~DAMP_HOOK_HOLD_FIRST_ITEM) return DAMP_ERR_INVALID_ARGUMENT;
    g_wait_ns.store(wait_limit_ns, std::memory_order_relaxed);
    g_hooks.store(hooks, std::memory_order_relaxed);
    return DAMP_OK;
}

size_t damp_calib_bytes(int H, int d_k) {
    if (H <= 0 || d_k <= 0) return 0;
    return (2 * (size_t)H * d_k + (size_t)H) * sizeof(double);
}

int damp_calib_accumulate(const damp_pool* pool, int n, const int32_t* slot_idx, int gate,
                          const float* alpha, double* acc, void* stream) {
    if (!pool || n < 0 || !pool->d.dev_buf) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    if (d.format != DAMP_FMT_FP32) return DAMP_ERR_INVALID_ARGUMENT;
    if (gate != DAMP_GATE_SCALAR && gate != DAMP_GATE_VECTOR) return DAMP_ERR_INVALID_ARGUMENT;
    if (n == 0) return DAMP_OK;
    if (!slot_idx || !alpha || !acc) return DAMP_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(slot_idx) & 3u) || (reinterpret_cast<uintptr_t>(alpha) & 3u) ||
        (reinterpret_cast<uintptr_t>(acc) & 7u))
        return DAMP_ERR_MISALIGNED;
    damp::CalibArgs a{};
    a.state = reinterpret_cast<const float*>(d.dev_buf + d.header_bytes);
    a.status = reinterpret_cast<uint32_t*>(d.dev_buf);
    a.slot_idx = slot_idx;
    a.alpha = alpha;
    a.acc = acc;
    a.n = n;
    a.H = d.H;
    a.n_slots = d.n_slots;
    a.gate = gate;
    a.d_k = d.d_k;
    a.d_v = d.d_v;
    return cuda_status(damp::launch_calib_accumulate(a, static_cast<cudaStream_t>(stream)));
}

static int calib_shape(int H, int d_k) {
    if (H <= 0 || d_k <= 0) return DAMP_ERR_INVALID_ARGUMENT;
    if (!dim_ok(d_k)) return DAMP_ERR_UNSUPPORTED;
    return DAMP_OK;
}

int damp_calib_select(int H, int d_k, int hp_rows, const double* acc, double* score,
                      uint16_t* hp_row_idx, void* stream) {
    int rc = calib_shape(H, d_k);
    if (rc) return rc;
    if (hp_rows < 0 || hp_rows > d_k || !acc || (hp_rows > 0 && !hp_row_idx))
        return DAMP_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(acc) & 7u) || (reinterpret_cast<uintptr_t>(score) & 7u) ||
        (reinterpret_cast<uintptr_t>(hp_row_idx) & 1u))
        return DAMP_ERR_MISALIGNED;
    return cuda_status(damp::launch_calib_select(acc, H, d_k, hp_rows, score, hp_row_idx,
                                                 static_cast<cudaStream_t>(stream)));
}

int damp_calib_select_budget(int H, int d_k, int budget, const double* acc, double* score,
                             uint8_t* is_fp16, int32_t* hp_per_head, void* stream) {
    int rc = calib_shape(H, d_k);
    if (rc) return rc;
    if (budget < 0 || (size_t)budget > (size_t)H * d_k || !acc || !score || !is_fp16 ||
        !hp_per_head)
        return DAMP_ERR_INVALID_ARGUMENT;
    if ((size_t)H * d_k > (size_t)0x7fffffff) return DAMP_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(acc) & 7u) || (reinterpret_cast<uintptr_t>(score) & 7u) ||
        (reinterpret_cast<uintptr_t>(hp_per_head) & 3u))
        return DAMP_ERR_MISALIGNED;
    return cuda_status(damp::launch_calib_select_budget(acc, H, d_k, budget, score, is_fp16,
                                                        hp_per_head,
                                                        static_cast<cudaStream_t>(stream)));
}

int damp_validate_slots(const int32_t* slot_idx, int n, int n_slots, int* bad_entry) {
    if (bad_entry) *bad_entry = -1;
    if (n < 0 || n_slots < 1 || (n > 0 && !slot_idx)) return DAMP_ERR_INVALID_ARGUMENT;
    std::vector<uint8_t> seen((size_t)n_slots, 0);
    for (int b = 0; b < n; ++b) {
        const int32_t s = slot_idx[b];
        if (s < 0) continue;
        if (s >= n_slots || seen[(size_t)s]) {
            if (bad_entry) *bad_entry = b;
            return DAMP_ERR_INVALID_ARGUMENT;
        }
        seen[(size_t)s] = 1;
    }
    return DAMP_OK;
}

int damp_pool_get_error(const damp_pool* pool, uint32_t* flags, int clear, void* stream) {
    if (!pool || !flags || !pool->d.dev_buf) return DAMP_ERR_INVALID_ARGUMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Wait for the work already queued by polling an event, with a deadline,
    // so that a stream that never drains is reported instead of waited on.
    cudaEvent_t ev;
    cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return DAMP_ERR_CUDA;
    e = cudaEventRecord(ev, s);
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::seconds(10);
    while (e == cudaSuccess) {
        const cudaError_t q = cudaEventQuery(ev);
        if (q == cudaSuccess) break;
        if (q != cudaErrorNotReady) {
            e = q;
            break;
        }
        if (std::chrono::steady_clock::now() > deadline) {
            cudaEventDestroy(ev);
            return DAMP_ERR_TIMEOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    cudaEventDestroy(ev);
    if (e != cudaSuccess) return DAMP_ERR_CUDA;
    uint32_t* st = reinterpret_cast<uint32_t*>(pool->d.dev_buf);
    uint32_t host = 0;
    e = cudaMemcpyAsync(&host, st, 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(st, 0, 4, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);   // the two tiny operations above
    if (e != cudaSuccess) return DAMP_ERR_CUDA;
    *flags = host;
    return DAMP_OK;
}

int damp_block_to_logical(const damp_pool* pool, int h, const void* block, float* scale,
                          uint16_t* half, int8_t* code, float* f32) {
    if (!pool || !block || h < 0 || h >= pool->d.H) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    const uint8_t* b = static_cast<const uint8_t*>(block);
    const int DK = d.d_k, DV = d.d_v;
    if (d.format == DAMP_FMT_FP32) {
        if (!f32) return DAMP_ERR_INVALID_ARGUMENT;
        memcpy(f32, b, (size_t)DK * DV * 4);
        return DAMP_OK;
    }
    if (!scale || !half || !code) return DAMP_ERR_INVALID_ARGUMENT;
    const uint32_t f16_off = d.host_heads[(size_t)h * 4 + 2], i8_off = d.host_heads[(size_t)h * 4 + 3];
    int r16 = 0, r8 = 0;
    for (int i = 0; i < DK; ++i) {
        if (is_fp16_row(d, h, i)) {
            scale[i] = 0.0f;
            const uint8_t* row = b + f16_off + (size_t)r16 * 2 * DV;
            for (int j = 0; j < DV; ++j) memcpy(half + (size_t)i * DV + j, row + damp::f16_pos(j, DV), 2);
            memset(code + (size_t)i * DV, 0, DV);
            ++r16;
        } else {
            memcpy(&scale[i], b + (size_t)r8 * 4, 4);
            memcpy(code + (size_t)i * DV, b + i8_off + (size_t)r8 * DV, DV);
            memset(half + (size_t)i * DV, 0, (size_t)2 * DV);
            ++r8;
        }
    }
    return DAMP_OK;
}

int damp_block_from_logical(const damp_pool* pool, int h, const float* scale,
                            const uint16_t* half, const int8_t* code, const float* f32,
                            void* block) {
    if (!pool || !block || h < 0 || h >= pool->d.H) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    uint8_t* b = static_cast<uint8_t*>(block);
    const int DK = d.d_k, DV = d.d_v;
    if (d.format == DAMP_FMT_FP32) {
        if (!f32) return DAMP_ERR_INVALID_ARGUMENT;
        memcpy(b, f32, (size_t)DK * DV * 4);
        return DAMP_OK;
    }
    if (!scale || !half || !code) return DAMP_ERR_INVALID_ARGUMENT;
    const uint32_t f16_off = d.host_heads[(size_t)h * 4 + 2], i8_off = d.host_heads[(size_t)h * 4 + 3];
    memset(b, 0, d.host_heads[(size_t)h * 4 + 1]);
    int r16 = 0, r8 = 0;
    for (int i = 0; i < DK; ++i) {
        if (is_fp16_row(d, h, i)) {
            uint8_t* row = b + f16_off + (size_t)r16 * 2 * DV;
            for (int j = 0; j < DV; ++j) memcpy(row + damp::f16_pos(j, DV), half + (size_t)i * DV + j, 2);
            ++r16;
        } else {
            memcpy(b + (size_t)r8 * 4, &scale[i], 4);
            memcpy(b + i8_off + (size_t)r8 * DV, code + (size_t)i * DV, DV);
            ++r8;
        }
    }
    return DAMP_OK;
}

int damp_pool_read_raw(const damp_pool* pool, int slot, int h, void* host_out) {
    if (!pool || !host_out || !pool->d.dev_buf) return DAMP_ERR_INVALID_ARGUMENT;
    const PoolDesc& d = pool->d;
    if (slot < 0 || slot >= d.n_slots || h < 0 || h >= d.H) return DAMP_ERR_INVALID_ARGUMENT;
    const uint32_t stride = d.host_heads[(size_t)h * 4 + 1];
    std::vector<uint8_t> raw(stride);
    const size_t off = d.header_bytes + (size_t)slot * d.slot_stride + d.host_heads[(size_t)h * 4];
    if (cudaMemcpy(raw.data(), d.dev_buf + off, stride, cudaMemcpyDeviceToHost) != cudaSuccess)
        return DAMP_ERR_CUDA;
    const size_t ne = (size_t)d.d_k * d.d_v;
    uint8_t* o = static_cast<uint8_t*>(host_out);
    if (d.format == DAMP_FMT_FP32)
        return damp_block_to_logical(pool, h, raw.data(), nullptr, nullptr, nullptr,
                                     reinterpret_cast<float*>(o));
    float* scale = reinterpret_cast<float*>(o);
    uint16_t* half = reinterpret_cast<uint16_t*>(o + 4 * (size_t)d.d_k);
    int8_t* code = reinterpret_cast<int8_t*>(o + 4 * (size_t)d.d_k + 2 * ne);
    return damp_block_to_logical(pool, h, raw.data(), scale, half, code, nullptr);
}

}  // extern "C"
