// noalloc.cu — moe_forward_noalloc: the expert FFN + combine without any
// device allocation.
//
// Some callers cannot call cudaMalloc: code running inside another
// framework's memory pool or allocator callback, embedders whose device
// memory is budgeted and accounted by someone else, or code paths that must
// not allocate while other streams are being captured.  For them this entry
// point keeps its scratch (the device status word and the SwiGLU activations
// h) in one file-scope device array of fixed size instead of a
// caller-supplied workspace.  The kernels are the same ones moe_forward runs,
// reading the experts from the contiguous weights' base address (no expert
// table is needed).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/moe_mxfp4.h"
#include "kernels.cuh"

namespace {

constexpr size_t kStatusOff = 0;
constexpr size_t kHOff = 256;
constexpr size_t kScratchBytes = kHOff + (size_t)MOE_NOALLOC_MAX_H_BYTES;
static_assert(kScratchBytes == MOE_NOALLOC_SCRATCH_BYTES, "scratch size as declared");

// The scratch itself: every GPU that loads this library holds it until exit.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct DeviceScratch {
    std::once_flag once;
    int rc = MOE_ERR_CUDA;
    uint8_t *addr = nullptr;  // device address of g_noalloc_scratch on this device
    int sms = 0;
};
DeviceScratch g_dev[kMaxDevices];

// Per device, once (thread-safe), with that device current: the symbol's
// device address and the SM count.
int scratch_for_current_device(uint8_t **base, int *sms) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    DeviceScratch &d = g_dev[dev];
    std::call_once(d.once, [&d, dev] {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            d.rc = MOE_ERR_CUDA;
            return;
        }
        if (major != 10) {
            d.rc = MOE_ERR_UNSUPPORTED;
            return;
        }
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            d.rc = MOE_ERR_CUDA;
            return;
        }
        d.sms = n;
        d.addr = static_cast<uint8_t *>(p);
        d.rc = MOE_OK;
    });
    if (d.rc != MOE_OK) return d.rc;
    *base = d.addr;
    *sms = d.sms;
    return MOE_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" int moe_forward_noalloc(int E, int H, int I, int top_k, const uint8_t *codes_u8,
                                   const uint8_t *scales_e8m0, const uint16_t *x, int T,
                                   const int32_t *topk_ids, const float *topk_w,
                                   const uint16_t *residual, uint16_t *y, void *stream) {
    if (E < 1 || H < 32 || I < 32 || H % 32 || I % 32 || H > 4096 || I > 4096) return MOE_ERR_ARG;
    if (top_k < 1 || top_k > moe::kMaxTopK || top_k > E || T < 1) return MOE_ERR_ARG;
    if ((size_t)T * top_k * I * 2 > (size_t)MOE_NOALLOC_MAX_H_BYTES) return MOE_ERR_WORKSPACE;
    if (!codes_u8 || !scales_e8m0 || !x || !topk_ids || !topk_w || !y || y == x) return MOE_ERR_ARG;
    if (!aligned16(codes_u8) || !aligned16(scales_e8m0) || !aligned16(x) || !aligned16(y) ||
        (residual && !aligned16(residual)))
        return MOE_ERR_ALIGN;
    if (!moe::decode_shape_supported(H, I)) return MOE_ERR_ARG;

    uint8_t *base = nullptr;
    int sms = 0;
    int rc = scratch_for_current_device(&base, &sms);
    if (rc != MOE_OK) return rc;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t mc = (size_t)I * H / 2, ms = (size_t)I * H / 32;
    if (ms % 16) return MOE_ERR_ALIGN;

    unsigned *d_status = reinterpret_cast<unsigned *>(base + kStatusOff);
    uint16_t *d_h = reinterpret_cast<uint16_t *>(base + kHOff);

    // same per-(token, slot) GEMV path as moe_forward, in token chunks sized so
    // that the down kernel's staged activations fit in shared memory
    int chunk = moe::kDecodeMaxT;
    while (chunk > 1 && moe::down_decode_smem(chunk, top_k, I, (chunk * H + sms - 1) / sms) >
                            moe::kDownSmemMax)
        --chunk;
    if (moe::down_decode_smem(1, top_k, I, (H + sms - 1) / sms) > moe::kDownSmemMax)
        return MOE_ERR_ARG;
    for (int t0 = 0; t0 < T; t0 += chunk) {
        const int Tc = (T - t0 < chunk) ? T - t0 : chunk;
        moe::GateUpParams g = {};
        g.table = nullptr;  // experts addressed from the contiguous base
        g.codes_base = codes_u8;
        g.scales_base = scales_e8m0;
        g.codes_stride = mc;
        g.scales_stride = ms;
        g.x = x + (size_t)t0 * H;
        g.x16 = nullptr;
        g.x16_exp = nullptr;
        g.ids = topk_ids + (size_t)t0 * top_k;
        g.logits = nullptr;
        g.ids_out = nullptr;
        g.w_out = nullptr;
        g.nslots = moe::gateup_tma_slots(H);
        g.h = d_h + (size_t)t0 * top_k * I;
        g.status = d_status;
        g.T = Tc;
        g.k = top_k;
        g.E = E;
        g.H = H;
        g.I = I;
        g.prefetch_down = 1;
        g.pf_codes = (uint32_t)(((mc + sms - 1) / sms + 15) / 16 * 16);
        g.pf_scales = (uint32_t)(((ms + sms - 1) / sms + 15) / 16 * 16);
        if (moe::launch_gateup_decode(g, sms, s, true) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        moe::DownParams d = {};
        d.table = nullptr;
        d.codes_base = codes_u8;
        d.scales_base = scales_e8m0;
        d.codes_stride = mc;
        d.scales_stride = ms;
        d.h = g.h;
        d.ids = g.ids;
        d.w = topk_w + (size_t)t0 * top_k;
        d.logits = nullptr;
        d.residual = residual ? residual + (size_t)t0 * H : nullptr;
        d.y = y + (size_t)t0 * H;
        d.o_keep = nullptr;
        d.status = d_status;
        d.T = Tc;
        d.k = top_k;
        d.E = E;
        d.H = H;
        d.I = I;
        const int rows = Tc * H;
        d.rows_per_cta = (rows + sms - 1) / sms;
        const int grid = (rows + d.rows_per_cta - 1) / d.rows_per_cta;
        if (moe::launch_down_decode(d, grid, s, true) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    }
    return MOE_OK;
}

extern "C" int moe_forward_noalloc_status(void *stream, unsigned *device_status) {
    if (!device_status) return MOE_ERR_ARG;
    uint8_t *base = nullptr;
    int sms = 0;
    int rc = scratch_for_current_device(&base, &sms);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned *d_status = reinterpret_cast<unsigned *>(base + kStatusOff);
    unsigned v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyAsync(&v, d_status, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(d_status, 0, sizeof v, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    *device_status = v;
    return MOE_OK;
}
