// damp_codec.cu -- pack (FP32 states -> pool blocks) and unpack (pool blocks
// -> FP32 states) kernels of libdamp.
//
// Pack is the hand-off from prefill (or a restore): the FP32 state is stored
// in the pool's format with the same codec the decode step uses when it
// requantizes (FP16 rows rounded to nearest even; INT8 rows with a per-row
// FP32 absmax scale).  Unpack is "STEPQuant ...", Appendix Table C2, step 1
// on its own: FP16 rows exactly, INT8 rows as fl(code * scale).
//
// Both use the decode step's thread tile (a 256-thread CTA holds 128/d
// units; a thread owns d/8 rows x 4 columns) and walk work items with a grid
// stride; they read and write global memory directly (coalesced 4/8/16-byte
// accesses per lane along a row).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "damp.h"
#include "damp_device.cuh"

namespace damp {
namespace {

constexpr int kCodecThreads = 256;

template <int D, bool QUANT, bool PACK, bool FP8>
__global__ void __launch_bounds__(kCodecThreads) codec_kernel(const CodecArgs a) {
    using G = Geo<D>;
    constexpr int RPT = G::RPT, UPI = G::UPI, LPR = G::LPR;
    __shared__ float rowbuf_all[UPI * 8 * 2 * RPT];
    const int tid = threadIdx.x;
    const int ui = tid / G::TPU, tu = tid % G::TPU;
    const int cg = tu % LPR, rg = tu / LPR, r0 = rg * RPT;
    float* rowbuf = rowbuf_all + (ui * 8 + rg) * 2 * RPT;
    const int n_units = a.n * a.H;

    for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
        const int u = item * UPI + ui;
        if (u >= n_units) continue;  // whole warps skip together (2d >= 32 threads per unit)
        const int b = u / a.H, h = u % a.H;
        const int slot = __ldg(a.slot_idx + b);
        float* st = a.state + (size_t)u * D * D;
        const bool ok = slot >= 0 && slot < a.n_slots;
        if (!ok && slot >= a.n_slots && tu == 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
        // this head's block: {offset in the slot, stride, FP16-row offset, INT8-row offset}
        const uint4 hb = __ldg(a.heads + h);
        uint8_t* blk = ok ? a.blocks + (size_t)slot * a.slot_stride + hb.x : nullptr;
        uint32_t bits = 0;
        int rank16 = 0;
        if (QUANT && ok) {
            const uint4 mw = __ldg(reinterpret_cast<const uint4*>(a.masks + (size_t)h * kMaskWords));
            row_formats<D>(mw, r0, bits, rank16);
        }
        float2 x[RPT][2];
        if constexpr (PACK) {
            if (!ok) continue;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float4 f =
                    __ldg(reinterpret_cast<const float4*>(st + (size_t)(r0 + i) * D + 4 * cg));
                x[i][0] = make_float2(f.x, f.y);
                x[i][1] = make_float2(f.z, f.w);
            }
            if constexpr (QUANT) {
                store_quant_tile<D, FP8>(blk, hb.z, hb.w, bits, rank16, r0, cg, x, rowbuf);
            } else {
#pragma unroll
                for (int i = 0; i < RPT; ++i)
                    *reinterpret_cast<float4*>(blk + ((size_t)(r0 + i) * D + 4 * cg) * 4) =
                        make_float4(x[i][0].x, x[i][0].y, x[i][1].x, x[i][1].y);
            }
        } else {
            if (!ok) {
#pragma unroll
                for (int i = 0; i < RPT; ++i)
                    *reinterpret_cast<float4*>(st + (size_t)(r0 + i) * D + 4 * cg) =
                        make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            if constexpr (QUANT) {
                load_tile_mask<D, FP8>(blk, hb.z, hb.w, bits, rank16, r0, cg, x);
            } else {
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const float4 f = *reinterpret_cast<const float4*>(
                        blk + ((size_t)(r0 + i) * D + 4 * cg) * 4);
                    x[i][0] = make_float2(f.x, f.y);
                    x[i][1] = make_float2(f.z, f.w);
                }
            }
#pragma unroll
            for (int i = 0; i < RPT; ++i)
                *reinterpret_cast<float4*>(st + (size_t)(r0 + i) * D + 4 * cg) =
                    make_float4(x[i][0].x, x[i][0].y, x[i][1].x, x[i][1].y);
        }
    }
}

template <int D, bool QUANT, bool PACK, bool FP8>
cudaError_t launch_codec_t(const CodecArgs& a, cudaStream_t stream) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int grid = std::max(1, std::min(a.n_items, sms * 8));
    codec_kernel<D, QUANT, PACK, FP8><<<grid, kCodecThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int D, bool PACK>
cudaError_t dispatch_d(int format, const CodecArgs& a, cudaStream_t s) {
    if (format == DAMP_FMT_FP32) return launch_codec_t<D, false, PACK, false>(a, s);
    if (format == DAMP_FMT_FP8_ROW) return launch_codec_t<D, true, PACK, true>(a, s);
    return launch_codec_t<D, true, PACK, false>(a, s);
}

// Square d in {16, 32, 64, 128}: the thread-tile kernel above (a.n_items
// counts units; an item holds 128/d of them); any other shape: the one-CTA-
// per-unit kernels of damp_decode_any.cu.
template <bool PACK>
cudaError_t dispatch(const PoolDesc& p, const CodecArgs& a0, cudaStream_t s) {
    CodecArgs a = a0;
    if (p.d_k != p.d_v || p.d_k > kMaxFastD || (p.d_k & (p.d_k - 1)))
        return PACK ? launch_pack_any(a, s) : launch_unpack_any(a, s);
    const int upi = kMaxFastD / p.d_k;
    a.n_items = (a.n_items + upi - 1) / upi;
    switch (p.d_k) {
        case 16: return dispatch_d<16, PACK>(p.format, a, s);
        case 32: return dispatch_d<32, PACK>(p.format, a, s);
        case 64: return dispatch_d<64, PACK>(p.format, a, s);
        case 128: return dispatch_d<128, PACK>(p.format, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_pack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream) {
    return dispatch<true>(p, a, stream);
}
cudaError_t launch_unpack(const PoolDesc& p, const CodecArgs& a, cudaStream_t stream) {
    return dispatch<false>(p, a, stream);
}

}  // namespace damp
