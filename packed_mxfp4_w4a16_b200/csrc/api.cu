// api.cu — host implementation of the C ABI declared in include/moe_mxfp4.h.
//
// The handle holds shapes, the device expert table (the persistent device
// pointer table of the model card's section "Direct reads from GPU-resident
// weights"), a device status word and the caller's workspace.  route/forward
// validate their arguments on the host and then only enqueue kernels: no
// allocation, no synchronisation, no weight copy, so a whole layer (or a whole
// stack of layers) can be captured in one CUDA graph (model card sections
// "Grouped top-4 expert execution" and "Shared capture stream").
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "../../include/moe_mxfp4.h"
#include "kernels.cuh"

struct moe_ctx {
    int E = 0, H = 0, I = 0, k = 0;
    int device = -1;
    int num_sms = 0;
    void *dblock = nullptr;               // device: ExpertPtrs[E], then status word
    moe::ExpertPtrs *d_table = nullptr;
    unsigned *d_status = nullptr;
    bool loaded = false;
    uint8_t *ws = nullptr;
    size_t ws_bytes = 0;
    int max_tokens = 0;
    bool kept = false;                    // last forward kept intermediates
    bool use_pdl = true;
    bool prefetch_down = true;
    int fusion = 0;                       // moe_layer_ex launch structure (moe_set_fusion)
    const uint8_t *codes_base = nullptr;   // set by moe_load_packed (contiguous layout)
    const uint8_t *scales_base = nullptr;
    int nv = 0;                           // NVFP4 weights (moe_load_packed_nvfp4)
    const float *gscale = nullptr;        // NVFP4: [E][2] multipliers (gate/up, down)
    int s8 = 0;                           // sym8 weights (moe_load_packed_sym8)
    bool s8_scales4 = false;              // sym8 scales 4-byte aligned (grouped products)
    moe::TcMapCache tc_maps;              // tensor maps of the bound codes (tcgen05 products)
};

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
    size_t counters, logits, h, o, x16, x16_exp;
    size_t hand_seq, hand_ack, hand_ent;  // fused-layer routing handoff
    size_t logit_ent;                     // fused-layer tagged logits
    size_t h_tag;                         // one-launch layer: tagged h
    size_t perm, offs, h16, h_exp;        // grouped path: sorted pairs, staged h
    size_t total;
};

WsLayout ws_layout(const moe_ctx *c, int maxT) {
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t o = off;
        off = align_up(off + n, 256);
        return o;
    };
    L.counters = take((size_t)maxT * sizeof(unsigned));
    L.logits = take((size_t)maxT * c->E * sizeof(float));
    L.h = take((size_t)maxT * c->k * c->I * 2);
    L.o = take((size_t)maxT * c->k * c->H * 2);
    L.x16 = take((size_t)maxT * c->H * 2);
    L.x16_exp = take((size_t)maxT * sizeof(int));
    L.hand_seq = take((size_t)moe::kHandMaxCtas * sizeof(unsigned));
    L.hand_ack = take((size_t)moe::kHandMaxCtas * sizeof(unsigned));
    L.hand_ent = take((size_t)moe::kHandMaxCtas * moe::kHandStride * 2 * sizeof(uint2));
    L.logit_ent = take((size_t)moe::kDecodeMaxT * moe::kFusedMaxE * sizeof(uint2));
    L.h_tag = take((size_t)maxT * c->k * c->I * sizeof(uint2));
    L.perm = take((size_t)maxT * c->k * sizeof(int));
    L.offs = take((size_t)(c->E + 1) * sizeof(int));
    L.h16 = take((size_t)maxT * c->k * c->I * 2);
    L.h_exp = take((size_t)maxT * c->k * sizeof(int));
    L.total = off;
    return L;
}

int check_device_ptr(const moe_ctx *c, const void *p, size_t align) {
    if (!p) return MOE_ERR_ARG;
    if (((uintptr_t)p) & (align - 1)) return MOE_ERR_ALIGN;
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_NOT_DEVICE;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return MOE_ERR_NOT_DEVICE;
    if (c && a.device != c->device) return MOE_ERR_NOT_DEVICE;
    return MOE_OK;
}

int current_device_ok(int *dev, int *sms) {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    int major = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (major != 10) return MOE_ERR_UNSUPPORTED;
    if (dev) *dev = d;
    if (sms) *sms = n;
    return MOE_OK;
}

int ensure_device_block(moe_ctx *c) {
    if (c->dblock) return MOE_OK;
    int rc = current_device_ok(&c->device, &c->num_sms);
    if (rc != MOE_OK) return rc;
    size_t tbytes = align_up(sizeof(moe::ExpertPtrs) * (size_t)c->E, 256);
    void *p = nullptr;
    if (cudaMalloc(&p, tbytes + 256) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (cudaMemset(p, 0, tbytes + 256) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(p);
        return MOE_ERR_CUDA;
    }
    c->dblock = p;
    c->d_table = reinterpret_cast<moe::ExpertPtrs *>(p);
    c->d_status = reinterpret_cast<unsigned *>(static_cast<uint8_t *>(p) + tbytes);
    return MOE_OK;
}

int upload_table(moe_ctx *c, const moe::ExpertPtrs *host_table) {
    cudaError_t e = cudaMemcpy(c->d_table, host_table, sizeof(moe::ExpertPtrs) * (size_t)c->E,
                               cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    c->loaded = true;
    return MOE_OK;
}

int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    cudaGetLastError();
    return MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

int moe_create(int E, int H, int I, int top_k, moe_handle_t *out) {
    if (!out) return MOE_ERR_ARG;
    *out = nullptr;
    if (E < 1 || E > 1024 || H < 32 || I < 32 || H % 32 || I % 32) return MOE_ERR_ARG;
    if (top_k < 1 || top_k > moe::kMaxTopK || top_k > E) return MOE_ERR_ARG;
    if (H > 4096 || I > 4096) return MOE_ERR_ARG;
    moe_ctx *c = new (std::nothrow) moe_ctx;
    if (!c) return MOE_ERR_ARG;
    c->E = E;
    c->H = H;
    c->I = I;
    c->k = top_k;
    *out = c;
    return MOE_OK;
}

int moe_destroy(moe_handle_t h) {
    if (!h) return MOE_OK;
    int rc = MOE_OK;
    if (h->dblock) {
        cudaDeviceSynchronize();
        rc = cuda_rc(cudaFree(h->dblock));
    }
    delete h;
    return rc;
}

int moe_load_packed(moe_handle_t h, const uint8_t *codes_u8, const uint8_t *scales_e8m0) {
    if (!h || !codes_u8 || !scales_e8m0) return MOE_ERR_ARG;
    int rc = ensure_device_block(h);
    if (rc != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, codes_u8, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, scales_e8m0, 16)) != MOE_OK) return rc;
    const size_t mc = (size_t)h->I * h->H / 2, ms = (size_t)h->I * h->H / 32;
    if (ms % 16) return MOE_ERR_ALIGN;  // every matrix must start 16-byte aligned
    moe::ExpertPtrs *t = new (std::nothrow) moe::ExpertPtrs[h->E];
    if (!t) return MOE_ERR_ARG;
    for (int e = 0; e < h->E; ++e)
        for (int m = 0; m < 3; ++m) {
            t[e].codes[m] = codes_u8 + ((size_t)e * 3 + m) * mc;
            t[e].scales[m] = scales_e8m0 + ((size_t)e * 3 + m) * ms;
        }
    rc = upload_table(h, t);
    delete[] t;
    if (rc == MOE_OK) {
        h->codes_base = codes_u8;
        h->scales_base = scales_e8m0;
        h->nv = 0;
        h->s8 = 0;
        h->gscale = nullptr;
    }
    return rc;
}

int moe_load_packed_nvfp4(moe_handle_t h, const uint8_t *codes_u8, const uint8_t *scales_e4m3,
                          const float *global_scales) {
    if (!h || !codes_u8 || !scales_e4m3 || !global_scales) return MOE_ERR_ARG;
    // the NVFP4 gate/up rows run on the bulk-copy kernel only
    if (!moe::gateup_tma_supported(h->H)) return MOE_ERR_ARG;
    int rc = ensure_device_block(h);
    if (rc != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, codes_u8, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, scales_e4m3, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, global_scales, 4)) != MOE_OK) return rc;
    const size_t mc = (size_t)h->I * h->H / 2, ms = (size_t)h->I * h->H / 16;
    if (ms % 16) return MOE_ERR_ALIGN;  // every matrix must start 16-byte aligned
    moe::ExpertPtrs *t = new (std::nothrow) moe::ExpertPtrs[h->E];
    if (!t) return MOE_ERR_ARG;
    for (int e = 0; e < h->E; ++e)
        for (int m = 0; m < 3; ++m) {
            t[e].codes[m] = codes_u8 + ((size_t)e * 3 + m) * mc;
            t[e].scales[m] = scales_e4m3 + ((size_t)e * 3 + m) * ms;
        }
    rc = upload_table(h, t);
    delete[] t;
    if (rc == MOE_OK) {
        h->codes_base = codes_u8;
        h->scales_base = scales_e4m3;
        h->nv = 1;
        h->s8 = 0;
        h->gscale = global_scales;
    }
    return rc;
}

int moe_load_packed_sym8(moe_handle_t h, const int8_t *codes_s8, const uint16_t *scales_f16) {
    if (!h || !codes_s8 || !scales_f16) return MOE_ERR_ARG;
    if (!moe::sym8_supported(h->H, h->I, h->k)) return MOE_ERR_ARG;
    int rc = ensure_device_block(h);
    if (rc != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, codes_s8, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, scales_f16, 2)) != MOE_OK) return rc;
    // one byte per weight; one 2-byte scale per 32 weights
    const size_t mc = (size_t)h->I * h->H, ms = (size_t)h->I * h->H / 16;
    const uint8_t *cb = reinterpret_cast<const uint8_t *>(codes_s8);
    const uint8_t *sb = reinterpret_cast<const uint8_t *>(scales_f16);
    moe::ExpertPtrs *t = new (std::nothrow) moe::ExpertPtrs[h->E];
    if (!t) return MOE_ERR_ARG;
    for (int e = 0; e < h->E; ++e)
        for (int m = 0; m < 3; ++m) {
            t[e].codes[m] = cb + ((size_t)e * 3 + m) * mc;
            t[e].scales[m] = sb + ((size_t)e * 3 + m) * ms;
        }
    rc = upload_table(h, t);
    delete[] t;
    if (rc == MOE_OK) {
        // the MXFP4 fast paths read codes_base; sym8 is reached through the table
        h->codes_base = h->scales_base = nullptr;
        h->nv = 0;
        h->s8 = 1;
        h->s8_scales4 = (reinterpret_cast<uintptr_t>(sb) & 3) == 0;
        h->gscale = nullptr;
    }
    return rc;
}

int moe_load_expert_table(moe_handle_t h, const uint8_t *const *codes_ptrs,
                          const uint8_t *const *scales_ptrs) {
    if (!h || !codes_ptrs || !scales_ptrs) return MOE_ERR_ARG;
    int rc = ensure_device_block(h);
    if (rc != MOE_OK) return rc;
    moe::ExpertPtrs *t = new (std::nothrow) moe::ExpertPtrs[h->E];
    if (!t) return MOE_ERR_ARG;
    for (int e = 0; e < h->E && rc == MOE_OK; ++e)
        for (int m = 0; m < 3 && rc == MOE_OK; ++m) {
            const uint8_t *cp = codes_ptrs[3 * e + m], *sp = scales_ptrs[3 * e + m];
            if ((rc = check_device_ptr(h, cp, 16)) != MOE_OK) break;
            if ((rc = check_device_ptr(h, sp, 16)) != MOE_OK) break;
            t[e].codes[m] = cp;
            t[e].scales[m] = sp;
        }
    if (rc == MOE_OK) rc = upload_table(h, t);
    delete[] t;
    if (rc == MOE_OK) {
        h->codes_base = h->scales_base = nullptr;
        h->nv = 0;
        h->s8 = 0;
        h->gscale = nullptr;
    }
    return rc;
}

int moe_workspace_bytes(moe_handle_t h, int max_tokens, size_t *bytes) {
    if (!h || !bytes || max_tokens < 1) return MOE_ERR_ARG;
    *bytes = ws_layout(h, max_tokens).total;
    return MOE_OK;
}

int moe_set_workspace(moe_handle_t h, void *workspace, size_t bytes, int max_tokens) {
    if (!h || !workspace || max_tokens < 1) return MOE_ERR_ARG;
    int rc = ensure_device_block(h);
    if (rc != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, workspace, 256)) != MOE_OK) return rc;
    if (bytes < ws_layout(h, max_tokens).total) return MOE_ERR_WORKSPACE;
    if ((rc = cuda_rc(cudaMemset(workspace, 0, bytes))) != MOE_OK) return rc;
    h->ws = static_cast<uint8_t *>(workspace);
    h->ws_bytes = bytes;
    h->max_tokens = max_tokens;
    h->kept = false;
    return MOE_OK;
}

int moe_route_ex(moe_handle_t h, const uint16_t *x, int T, const uint16_t *router_w,
                 const float *router_bias, unsigned flags, uint16_t *x_norm, float *logits,
                 int32_t *topk_ids, float *topk_w, void *stream) {
    if (!h || T < 1) return MOE_ERR_ARG;
    if (flags & ~(MOE_ROUTE_RMSNORM | MOE_ROUTE_SIGMOID)) return MOE_ERR_ARG;
    const bool norm = flags & MOE_ROUTE_RMSNORM;
    if (norm != (x_norm != nullptr)) return MOE_ERR_ARG;
    if (!h->ws) return MOE_ERR_NOT_LOADED;
    if (T > h->max_tokens) return MOE_ERR_WORKSPACE;
    int rc;
    if ((rc = check_device_ptr(h, x, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, router_w, 16)) != MOE_OK) return rc;
    if (router_bias && (rc = check_device_ptr(h, router_bias, 4)) != MOE_OK) return rc;
    if (norm && (rc = check_device_ptr(h, x_norm, 16)) != MOE_OK) return rc;
    if (logits && (rc = check_device_ptr(h, logits, 4)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, topk_ids, 4)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, topk_w, 4)) != MOE_OK) return rc;
    const WsLayout L = ws_layout(h, h->max_tokens);
    moe::RouteParams p;
    p.x = x;
    p.wr = router_w;
    p.bias = router_bias;
    p.x_norm = x_norm;
    p.logits_ws = reinterpret_cast<float *>(h->ws + L.logits);
    p.logits_out = logits;
    p.ids = topk_ids;
    p.w = topk_w;
    p.counters = reinterpret_cast<unsigned *>(h->ws + L.counters);
    p.T = T;
    p.E = h->E;
    p.H = h->H;
    p.k = h->k;
    p.rmsnorm = norm ? 1 : 0;
    p.sigmoid = (flags & MOE_ROUTE_SIGMOID) ? 1 : 0;
    p.eps = 1e-6f;
    p.x16 = nullptr;
    p.x16_exp = nullptr;
    return cuda_rc(moe::launch_route(p, static_cast<cudaStream_t>(stream), h->use_pdl));
}

int moe_route(moe_handle_t h, const uint16_t *x, int T, const uint16_t *router_w,
              const float *router_bias, int32_t *topk_ids, float *topk_w, void *stream) {
    return moe_route_ex(h, x, T, router_w, router_bias, 0u, nullptr, nullptr, topk_ids, topk_w,
                        stream);
}

int moe_forward_ex(moe_handle_t h, const uint16_t *x, int T, const int32_t *topk_ids,
                   const float *topk_w, const uint16_t *residual, uint16_t *y, unsigned flags,
                   void *stream) {
    if (!h || T < 1) return MOE_ERR_ARG;
    const unsigned known = MOE_FWD_KEEP_INTERMEDIATES | MOE_FWD_FORCE_DECODE |
                           MOE_FWD_FORCE_GROUPED | MOE_FWD_PHASE_GATEUP | MOE_FWD_PHASE_DOWN |
                           MOE_FWD_FORCE_TCGEN05 | MOE_FWD_FORCE_MMA;
    if (flags & ~known) return MOE_ERR_ARG;
    if ((flags & MOE_FWD_FORCE_TCGEN05) && (flags & MOE_FWD_FORCE_MMA)) return MOE_ERR_ARG;
    if (flags & MOE_FWD_FORCE_MMA) {
        if (flags & MOE_FWD_FORCE_DECODE) return MOE_ERR_ARG;
        flags |= MOE_FWD_FORCE_GROUPED;
    }
    if (flags & MOE_FWD_FORCE_TCGEN05) {
        if (flags & MOE_FWD_FORCE_DECODE) return MOE_ERR_ARG;
        if (h->s8 || !h->codes_base || !moe::grouped_tc_supported(h->H, h->I, h->nv))
            return MOE_ERR_ARG;
        flags |= MOE_FWD_FORCE_GROUPED;
    }
    if ((flags & MOE_FWD_FORCE_DECODE) && (flags & MOE_FWD_FORCE_GROUPED)) return MOE_ERR_ARG;
    if ((flags & MOE_FWD_PHASE_GATEUP) && (flags & MOE_FWD_PHASE_DOWN)) return MOE_ERR_ARG;
    const bool run_gu = !(flags & MOE_FWD_PHASE_DOWN);
    const bool run_dn = !(flags & MOE_FWD_PHASE_GATEUP);
    if (!h->loaded || !h->ws) return MOE_ERR_NOT_LOADED;
    if (T > h->max_tokens) return MOE_ERR_WORKSPACE;
    int rc;
    if ((rc = check_device_ptr(h, x, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, topk_ids, 4)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, topk_w, 4)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, y, 16)) != MOE_OK) return rc;
    if (residual && (rc = check_device_ptr(h, residual, 16)) != MOE_OK) return rc;
    if (y == x) return MOE_ERR_ARG;

    const WsLayout L = ws_layout(h, h->max_tokens);
    const bool keep = flags & MOE_FWD_KEEP_INTERMEDIATES;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint16_t *hbuf = reinterpret_cast<uint16_t *>(h->ws + L.h);
    uint16_t *obuf = reinterpret_cast<uint16_t *>(h->ws + L.o);

    // (token, expert)-sorted grouped path on the tensor cores: batches beyond
    // the decode sizes, or when asked (the phase flags time the decode path);
    // sym8 weights need their scales 4-byte aligned there
    const bool phase = flags & (MOE_FWD_PHASE_GATEUP | MOE_FWD_PHASE_DOWN);
    const bool grouped = !phase && !(flags & MOE_FWD_FORCE_DECODE) &&
                         (T > moe::kDecodeMaxT || (flags & MOE_FWD_FORCE_GROUPED)) &&
                         (!h->s8 || h->s8_scales4) &&
                         moe::grouped_supported(h->E, h->H, h->I, h->nv, h->s8);
    if ((flags & MOE_FWD_FORCE_GROUPED) && !grouped) return MOE_ERR_ARG;

    if (h->s8 && !grouped) {
        // sym8 experts off the grouped path: the per-(token, slot) GEMVs of
        // sym8.cu
        const int chunk = moe::sym8_max_chunk(h->H, h->I, h->k);
        for (int t0 = 0; t0 < T; t0 += chunk) {
            const int Tc = (T - t0 < chunk) ? T - t0 : chunk;
            moe::Sym8Params p = {};
            p.table = h->d_table;
            p.x = x + (size_t)t0 * h->H;
            p.ids = topk_ids + (size_t)t0 * h->k;
            p.w = topk_w + (size_t)t0 * h->k;
            p.residual = residual ? residual + (size_t)t0 * h->H : nullptr;
            p.y = y + (size_t)t0 * h->H;
            p.h = hbuf + (size_t)t0 * h->k * h->I;
            p.o_keep = keep ? obuf + (size_t)t0 * h->k * h->H : nullptr;
            p.status = h->d_status;
            p.T = Tc;
            p.E = h->E;
            p.H = h->H;
            p.I = h->I;
            p.k = h->k;
            if ((rc = cuda_rc(moe::launch_sym8(p, h->num_sms, run_gu, run_dn, s, h->use_pdl))) !=
                MOE_OK)
                return rc;
        }
        h->kept = keep;
        return MOE_OK;
    }
    if (!h->s8 && !moe::decode_shape_supported(h->H, h->I)) return MOE_ERR_ARG;

    if (grouped) {
        for (int t0 = 0; t0 < T; t0 += moe::kGroupedMaxT) {
            const int Tc = (T - t0 < moe::kGroupedMaxT) ? T - t0 : moe::kGroupedMaxT;
            moe::GroupedParams gp = {};
            gp.table = h->d_table;
            gp.codes_base = h->codes_base;
            gp.scales_base = h->scales_base;
            gp.codes_stride = (size_t)h->I * h->H / 2;
            gp.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
            gp.nv = h->nv;
            gp.s8 = h->s8;
            gp.gscale = h->gscale;
            gp.tc_maps = &h->tc_maps;
            gp.x = x + (size_t)t0 * h->H;
            gp.ids = topk_ids + (size_t)t0 * h->k;
            gp.w = topk_w + (size_t)t0 * h->k;
            gp.residual = residual ? residual + (size_t)t0 * h->H : nullptr;
            gp.y = y + (size_t)t0 * h->H;
            gp.o_keep = nullptr;  // o itself lands in the workspace buffer kept below
            gp.perm = reinterpret_cast<int *>(h->ws + L.perm);
            gp.offs = reinterpret_cast<int *>(h->ws + L.offs);
            gp.x16 = reinterpret_cast<uint32_t *>(h->ws + L.x16);
            gp.x_exp = reinterpret_cast<int *>(h->ws + L.x16_exp);
            gp.h = hbuf + (size_t)t0 * h->k * h->I;
            gp.h16 = reinterpret_cast<uint32_t *>(h->ws + L.h16);
            gp.h_exp = reinterpret_cast<int *>(h->ws + L.h_exp);
            gp.o = obuf + (size_t)t0 * h->k * h->H;
            gp.status = h->d_status;
            gp.T = Tc;
            gp.k = h->k;
            gp.E = h->E;
            gp.H = h->H;
            gp.I = h->I;
            // tcgen05 when the groups are large enough to amortise a CTA's
            // dequantised tiles over its token passes
            const bool tc_ok = !h->s8 && h->codes_base &&
                               moe::grouped_tc_supported(h->H, h->I, h->nv);
            gp.tcgen05 = (flags & MOE_FWD_FORCE_TCGEN05) ||
                         (!(flags & MOE_FWD_FORCE_MMA) && tc_ok &&
                          (long long)Tc * h->k >= (long long)moe::kTcAutoGroup * h->E);
            if ((rc = cuda_rc(moe::launch_grouped(gp, s, h->use_pdl))) != MOE_OK) return rc;
        }
        h->kept = keep;
        return MOE_OK;
    }

    // per-(token, slot) GEMV path, in chunks of up to kDecodeMaxT tokens (fewer
    // when the staged activations of a chunk would not fit in shared memory)
    int chunk = moe::kDecodeMaxT;
    while (chunk > 1 && (moe::gateup_decode_smem(chunk, h->H) > moe::kDownSmemMax ||
                         moe::down_decode_smem(chunk, h->k, h->I,
                                               (chunk * h->H + h->num_sms - 1) / h->num_sms) >
                             moe::kDownSmemMax))
        --chunk;
    if (moe::down_decode_smem(1, h->k, h->I, (h->H + h->num_sms - 1) / h->num_sms) >
        moe::kDownSmemMax)
        return MOE_ERR_ARG;
    for (int t0 = 0; t0 < T; t0 += chunk) {
        const int Tc = (T - t0 < chunk) ? T - t0 : chunk;
        moe::GateUpParams g = {};
        g.table = h->d_table;
        g.codes_base = h->codes_base;
        g.scales_base = h->scales_base;
        g.codes_stride = (size_t)h->I * h->H / 2;
        g.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
        g.x = x + (size_t)t0 * h->H;
        g.x16 = nullptr;
        g.x16_exp = nullptr;
        g.ids = topk_ids + (size_t)t0 * h->k;
        g.logits = nullptr;
        g.ids_out = nullptr;
        g.w_out = nullptr;
        g.nslots = moe::gateup_tma_slots(h->H, h->nv);
        g.nv = h->nv;
        g.gscale = h->gscale;
        g.h = hbuf + (size_t)t0 * h->k * h->I;
        g.status = h->d_status;
        g.T = Tc;
        g.k = h->k;
        g.E = h->E;
        g.H = h->H;
        g.I = h->I;
        g.prefetch_down = h->prefetch_down ? 1 : 0;
        {
            const size_t mc = (size_t)h->H * h->I / 2, ms = (size_t)h->H * h->I / 32;
            const size_t n = (size_t)h->num_sms;
            g.pf_codes = (uint32_t)(((mc + n - 1) / n + 15) / 16 * 16);
            g.pf_scales = (uint32_t)(((ms + n - 1) / n + 15) / 16 * 16);
        }
        if (run_gu &&
            (rc = cuda_rc(moe::launch_gateup_decode(g, h->num_sms, s, h->use_pdl))) != MOE_OK)
            return rc;

        moe::DownParams d = {};
        d.table = h->d_table;
        d.codes_base = h->codes_base;
        d.scales_base = h->scales_base;
        d.codes_stride = (size_t)h->I * h->H / 2;
        d.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
        d.h = g.h;
        d.ids = g.ids;
        d.w = topk_w + (size_t)t0 * h->k;
        d.logits = nullptr;
        d.residual = residual ? residual + (size_t)t0 * h->H : nullptr;
        d.y = y + (size_t)t0 * h->H;
        d.o_keep = keep ? obuf + (size_t)t0 * h->k * h->H : nullptr;
        d.status = h->d_status;
        d.T = Tc;
        d.k = h->k;
        d.E = h->E;
        d.H = h->H;
        d.I = h->I;
        const int rows = Tc * h->H;
        d.rows_per_cta = (rows + h->num_sms - 1) / h->num_sms;
        d.nv = h->nv;
        d.gscale = h->gscale;
        const int grid = (rows + d.rows_per_cta - 1) / d.rows_per_cta;
        if (run_dn && (rc = cuda_rc(moe::launch_down_decode(d, grid, s, h->use_pdl))) != MOE_OK)
            return rc;
    }
    h->kept = keep;
    return MOE_OK;
}

int moe_forward(moe_handle_t h, const uint16_t *x, int T, const int32_t *topk_ids,
                const float *topk_w, uint16_t *y, void *stream) {
    return moe_forward_ex(h, x, T, topk_ids, topk_w, nullptr, y, 0u, stream);
}

int moe_layer_ex(moe_handle_t h, const uint16_t *x, int T, const uint16_t *router_w,
                 const float *router_bias, unsigned route_flags, uint16_t *x_norm,
                 float *logits, int32_t *topk_ids, float *topk_w, const uint16_t *residual,
                 uint16_t *y, unsigned fwd_flags, void *stream) {
    if (!h || T < 1) return MOE_ERR_ARG;
    if (route_flags & ~(MOE_ROUTE_RMSNORM | MOE_ROUTE_SIGMOID)) return MOE_ERR_ARG;
    if (fwd_flags & ~MOE_FWD_KEEP_INTERMEDIATES) return MOE_ERR_ARG;
    const bool norm = route_flags & MOE_ROUTE_RMSNORM;
    if (norm != (x_norm != nullptr)) return MOE_ERR_ARG;
    if (!h->loaded || !h->ws) return MOE_ERR_NOT_LOADED;
    if (T > h->max_tokens) return MOE_ERR_WORKSPACE;
    int rc;
    if ((rc = check_device_ptr(h, x, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, router_w, 16)) != MOE_OK) return rc;
    if (router_bias && (rc = check_device_ptr(h, router_bias, 4)) != MOE_OK) return rc;
    if (norm && (rc = check_device_ptr(h, x_norm, 16)) != MOE_OK) return rc;
    if (logits && (rc = check_device_ptr(h, logits, 4)) != MOE_OK) return rc;
    if (topk_ids && (rc = check_device_ptr(h, topk_ids, 4)) != MOE_OK) return rc;
    if (topk_w && (rc = check_device_ptr(h, topk_w, 4)) != MOE_OK) return rc;
    if (residual && (rc = check_device_ptr(h, residual, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(h, y, 16)) != MOE_OK) return rc;
    if (norm && (x_norm == x || x_norm == y)) return MOE_ERR_ARG;
    if (!moe::decode_shape_supported(h->H, h->I)) return MOE_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(h, h->max_tokens);
    float *lg = reinterpret_cast<float *>(h->ws + L.logits);

    if (h->s8 && !(route_flags & MOE_ROUTE_SIGMOID) && T <= moe::sym8_max_chunk(h->H, h->I, h->k)) {
        // sym8 experts, one chunk of tokens, softmax scoring: the router
        // kernel writes the logits, and each sym8 kernel takes the top-k of
        // them itself (gate/up CTA 0 writes the routing out): three launches
        if (!topk_ids || !topk_w) return MOE_ERR_ARG;
        moe::RouteParams rp = {};
        rp.x = x;
        rp.wr = router_w;
        rp.bias = router_bias;
        rp.x_norm = x_norm;
        rp.logits_ws = lg;
        rp.logits_out = logits;
        rp.T = T;
        rp.E = h->E;
        rp.H = h->H;
        rp.k = h->k;
        rp.rmsnorm = norm ? 1 : 0;
        rp.eps = 1e-6f;
        rp.x16 = reinterpret_cast<uint32_t *>(h->ws + L.x16);
        rp.x16_exp = reinterpret_cast<int *>(h->ws + L.x16_exp);
        if ((rc = cuda_rc(moe::launch_route_logits(rp, s, h->use_pdl))) != MOE_OK) return rc;
        const bool keep = fwd_flags & MOE_FWD_KEEP_INTERMEDIATES;
        moe::Sym8Params p = {};
        p.table = h->d_table;
        p.x = norm ? x_norm : x;
        p.logits = lg;
        p.ids_out = topk_ids;
        p.w_out = topk_w;
        p.residual = residual;
        p.y = y;
        p.h = reinterpret_cast<uint16_t *>(h->ws + L.h);
        p.o_keep = keep ? reinterpret_cast<uint16_t *>(h->ws + L.o) : nullptr;
        p.status = h->d_status;
        p.T = T;
        p.E = h->E;
        p.H = h->H;
        p.I = h->I;
        p.k = h->k;
        if ((rc = cuda_rc(moe::launch_sym8(p, h->num_sms, true, true, s, h->use_pdl))) != MOE_OK)
            return rc;
        h->kept = keep;
        return MOE_OK;
    }
    if (T > moe::kDecodeMaxT || (route_flags & MOE_ROUTE_SIGMOID) || h->s8) {
        // many tokens, sigmoid scoring (the fused launch structures select
        // by softmax scoring only) or sym8 experts: explicit routing, then
        // the forward on the given ids
        int32_t *ids = topk_ids;
        float *w = topk_w;
        if (!ids || !w) return MOE_ERR_ARG;
        if ((rc = moe_route_ex(h, x, T, router_w, router_bias, route_flags, x_norm, logits, ids,
                               w, stream)) != MOE_OK)
            return rc;
        return moe_forward_ex(h, norm ? x_norm : x, T, ids, w, residual, y, fwd_flags, stream);
    }

    const bool keep = fwd_flags & MOE_FWD_KEEP_INTERMEDIATES;
    const int G = h->num_sms;
    size_t fsmem = 0;
    int fslots = 0;
    unsigned fregion = 0;
    const int frows = (T * h->H + G - 1) / G;
    unsigned fdown = 0;
    int lrows = 0;
    // the fused launch structures run MXFP4 weights only
    const bool mx = !h->nv && !h->s8;
    const bool whole = mx && h->fusion >= MOE_FUSION_LAYER && !keep &&
                       moe::layer_plan(T, h->E, h->H, h->I, h->k, G, &fsmem, &fslots, &fregion,
                                       &fdown, &lrows);
    if (whole || (mx && h->fusion >= MOE_FUSION_ROUTER &&
                  moe::layer_gateup_plan(T, h->E, h->H, G, &fsmem, &fslots, &fregion) &&
                  moe::down_decode_smem(T, h->k, h->I, frows) <= moe::kDownSmemMax)) {
        // router + gate/up in one launch, then the down kernel on the same grid
        // size (the routing handoff is per CTA index)
        moe::RouteHandoff hand;
        hand.seq = reinterpret_cast<unsigned *>(h->ws + L.hand_seq);
        hand.ack = reinterpret_cast<unsigned *>(h->ws + L.hand_ack);
        hand.ent = reinterpret_cast<uint2 *>(h->ws + L.hand_ent);
        moe::GateUpParams g = {};
        g.table = h->d_table;
        g.codes_base = h->codes_base;
        g.scales_base = h->scales_base;
        g.codes_stride = (size_t)h->I * h->H / 2;
        g.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
        g.x = norm ? x_norm : x;
        g.x16 = nullptr;
        g.x16_exp = nullptr;
        g.ids = nullptr;
        g.logits = nullptr;
        g.ids_out = topk_ids;
        g.w_out = topk_w;
        g.h = reinterpret_cast<uint16_t *>(h->ws + L.h);
        g.status = h->d_status;
        g.T = T;
        g.k = h->k;
        g.E = h->E;
        g.H = h->H;
        g.I = h->I;
        // the one-launch layer copies its down rows into shared memory itself
        g.prefetch_down = (h->prefetch_down && !whole) ? 1 : 0;
        {
            const size_t mc = (size_t)h->H * h->I / 2, ms = (size_t)h->H * h->I / 32;
            g.pf_codes = (uint32_t)(((mc + G - 1) / G + 15) / 16 * 16);
            g.pf_scales = (uint32_t)(((ms + G - 1) / G + 15) / 16 * 16);
        }
        g.nslots = fslots;
        moe::FusedRouteParams fr;
        fr.xr = x;
        fr.wr = router_w;
        fr.bias = router_bias;
        fr.x_norm = norm ? x_norm : nullptr;
        fr.logits_out = logits;
        fr.logit_ent = reinterpret_cast<uint2 *>(h->ws + L.logit_ent);
        fr.hand = hand;
        fr.rmsnorm = norm ? 1 : 0;
        fr.eps = 1e-6f;
        fr.region_bytes = fregion;
        if (whole) {
            // router + gate/up + down + combine in one launch
            moe::LayerDownParams dp = {};
            dp.residual = residual;
            dp.y = y;
            dp.h_tag = reinterpret_cast<uint2 *>(h->ws + L.h_tag);
            dp.rows_per_cta = lrows;
            dp.down_off = fdown;
            if ((rc = cuda_rc(moe::launch_layer(g, fr, dp, G, fsmem, s, h->use_pdl))) != MOE_OK)
                return rc;
            h->kept = false;
            return MOE_OK;
        }
        if ((rc = cuda_rc(moe::launch_layer_gateup(g, fr, G, fsmem, s, h->use_pdl))) != MOE_OK)
            return rc;
        moe::DownParams d = {};
        d.table = h->d_table;
        d.codes_base = h->codes_base;
        d.scales_base = h->scales_base;
        d.codes_stride = g.codes_stride;
        d.scales_stride = g.scales_stride;
        d.h = g.h;
        d.ids = nullptr;
        d.w = nullptr;
        d.logits = nullptr;
        d.hand = hand;
        d.residual = residual;
        d.y = y;
        d.o_keep = keep ? reinterpret_cast<uint16_t *>(h->ws + L.o) : nullptr;
        d.status = h->d_status;
        d.T = T;
        d.k = h->k;
        d.E = h->E;
        d.H = h->H;
        d.I = h->I;
        d.rows_per_cta = frows;
        if ((rc = cuda_rc(moe::launch_down_decode(d, G, s, h->use_pdl))) != MOE_OK) return rc;
        h->kept = keep;
        return MOE_OK;
    }

    moe::RouteParams rp;
    rp.sigmoid = 0;
    rp.x = x;
    rp.wr = router_w;
    rp.bias = router_bias;
    rp.x_norm = x_norm;
    rp.logits_ws = lg;
    rp.logits_out = logits;
    rp.ids = nullptr;
    rp.w = nullptr;
    rp.counters = nullptr;
    rp.T = T;
    rp.E = h->E;
    rp.H = h->H;
    rp.k = h->k;
    rp.rmsnorm = norm ? 1 : 0;
    rp.eps = 1e-6f;
    rp.x16 = reinterpret_cast<uint32_t *>(h->ws + L.x16);
    rp.x16_exp = reinterpret_cast<int *>(h->ws + L.x16_exp);
    if ((rc = cuda_rc(moe::launch_route_logits(rp, s, h->use_pdl))) != MOE_OK) return rc;

    moe::GateUpParams g = {};
    g.table = h->d_table;
    g.codes_base = h->codes_base;
    g.scales_base = h->scales_base;
    g.codes_stride = (size_t)h->I * h->H / 2;
    g.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
    g.x = norm ? x_norm : x;
    g.x16 = rp.x16;
    g.x16_exp = rp.x16_exp;
    g.ids = nullptr;
    g.logits = lg;
    g.ids_out = topk_ids;
    g.w_out = topk_w;
    g.h = reinterpret_cast<uint16_t *>(h->ws + L.h);
    g.status = h->d_status;
    g.T = T;
    g.k = h->k;
    g.E = h->E;
    g.H = h->H;
    g.I = h->I;
    g.prefetch_down = h->prefetch_down ? 1 : 0;
    {
        const size_t mc = (size_t)h->H * h->I / 2, ms = (size_t)h->H * h->I / 32;
        const size_t n = (size_t)h->num_sms;
        g.pf_codes = (uint32_t)(((mc + n - 1) / n + 15) / 16 * 16);
        g.pf_scales = (uint32_t)(((ms + n - 1) / n + 15) / 16 * 16);
    }
    g.nslots = moe::gateup_tma_slots(h->H, h->nv);
    g.nv = h->nv;
    g.gscale = h->gscale;
    if ((rc = cuda_rc(moe::launch_gateup_decode(g, h->num_sms, s, h->use_pdl))) != MOE_OK)
        return rc;

    moe::DownParams d = {};
    d.table = h->d_table;
    d.codes_base = h->codes_base;
    d.scales_base = h->scales_base;
    d.codes_stride = (size_t)h->I * h->H / 2;
    d.scales_stride = (size_t)h->I * h->H / (h->nv ? 16 : 32);
    d.h = g.h;
    d.ids = nullptr;
    d.w = nullptr;
    d.logits = lg;
    d.residual = residual;
    d.y = y;
    d.o_keep = keep ? reinterpret_cast<uint16_t *>(h->ws + L.o) : nullptr;
    d.status = h->d_status;
    d.T = T;
    d.k = h->k;
    d.E = h->E;
    d.H = h->H;
    d.I = h->I;
    const int rows = T * h->H;
    d.rows_per_cta = (rows + h->num_sms - 1) / h->num_sms;
    d.nv = h->nv;
    d.gscale = h->gscale;
    const int grid = (rows + d.rows_per_cta - 1) / d.rows_per_cta;
    if ((rc = cuda_rc(moe::launch_down_decode(d, grid, s, h->use_pdl))) != MOE_OK) return rc;
    h->kept = keep;
    return MOE_OK;
}

int moe_get_intermediates(moe_handle_t h, const uint16_t **h_out, const uint16_t **o_out) {
    if (!h || !h_out || !o_out) return MOE_ERR_ARG;
    if (!h->ws || !h->kept) return MOE_ERR_NOT_LOADED;
    const WsLayout L = ws_layout(h, h->max_tokens);
    *h_out = reinterpret_cast<const uint16_t *>(h->ws + L.h);
    *o_out = reinterpret_cast<const uint16_t *>(h->ws + L.o);
    return MOE_OK;
}

int moe_get_status(moe_handle_t h, unsigned *device_status) {
    if (!h || !device_status) return MOE_ERR_ARG;
    if (!h->dblock) return MOE_ERR_NOT_LOADED;
    int rc;
    if ((rc = cuda_rc(cudaDeviceSynchronize())) != MOE_OK) return rc;
    unsigned v = 0;
    if ((rc = cuda_rc(cudaMemcpy(&v, h->d_status, sizeof v, cudaMemcpyDeviceToHost))) != MOE_OK)
        return rc;
    if ((rc = cuda_rc(cudaMemset(h->d_status, 0, sizeof v))) != MOE_OK) return rc;
    *device_status = v;
    return MOE_OK;
}

int moe_get_status_stream(moe_handle_t h, void *stream, unsigned *device_status) {
    if (!h || !device_status) return MOE_ERR_ARG;
    if (!h->dblock) return MOE_ERR_NOT_LOADED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc;
    unsigned v = 0;
    // read and clear on the caller's stream, after the work queued on it
    if ((rc = cuda_rc(cudaMemcpyAsync(&v, h->d_status, sizeof v, cudaMemcpyDeviceToHost, s))) !=
        MOE_OK)
        return rc;
    if ((rc = cuda_rc(cudaMemsetAsync(h->d_status, 0, sizeof v, s))) != MOE_OK) return rc;
    if ((rc = cuda_rc(cudaStreamSynchronize(s))) != MOE_OK) return rc;
    *device_status = v;
    return MOE_OK;
}

int moe_bytes_per_expert(moe_handle_t h, size_t *bytes) {
    if (!h || !bytes) return MOE_ERR_ARG;
    *bytes = h->s8   ? (size_t)3 * h->I * h->H + (size_t)3 * h->I * h->H / 16
             : h->nv ? (size_t)3 * h->I * h->H / 2 + (size_t)3 * h->I * h->H / 16 + 2 * sizeof(float)
                     : (size_t)3 * h->I * h->H / 2 + (size_t)3 * h->I * h->H / 32;
    return MOE_OK;
}

int moe_set_tuning(moe_handle_t h, int use_pdl, int prefetch_down) {
    if (!h) return MOE_ERR_ARG;
    h->use_pdl = use_pdl != 0;
    h->prefetch_down = prefetch_down != 0;
    return MOE_OK;
}

int moe_set_fusion(moe_handle_t h, int mode) {
    if (!h || mode < MOE_FUSION_NONE || mode > MOE_FUSION_LAYER) return MOE_ERR_ARG;
    h->fusion = mode;
    return MOE_OK;
}

// ------------------------------------------------------------ stacks --

}  // extern "C"

struct moe_stack_ctx {
    int L = 0, E = 0, H = 0, I = 0, k = 0;
    int nv = 0;  // NVFP4 layers
    int device = -1;
    int num_sms = 0;
    uint8_t *ws = nullptr;
    size_t ws_bytes = 0;
    int spin_limit = moe::kMaxSpin;
    unsigned long long *trace = nullptr;
    moe::StackPlan plan = {};
    moe::StackLayer layer[moe::kStackMaxLayers] = {};
};

namespace {

struct StackWs {
    size_t x_tag, lg_tag, h_tag, seq, abort, status, total;
};

StackWs stack_ws_layout(const moe_stack_ctx *s) {
    StackWs W;
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t o = off;
        off = align_up(off + n, 256);
        return o;
    };
    // tagged words spread one 4-word piece (or one logit) per 128-byte line
    // (moe::kStkLine): see the stack kernel's exchange layout
    W.x_tag = take((size_t)s->H / 8 * moe::kStkLine);
    W.lg_tag = take((size_t)s->E * moe::kStkLine);
    W.h_tag = take((size_t)s->k * s->I / 8 * moe::kStkLine);
    W.seq = take((size_t)s->num_sms * sizeof(unsigned));
    W.abort = take(sizeof(unsigned));
    W.status = take(sizeof(unsigned));
    W.total = off;
    return W;
}

}  // namespace

extern "C" {

int moe_stack_create(const moe_handle_t *layers, int n_layers, const uint16_t *const *router_w,
                     const float *const *router_bias, moe_stack_t *out) {
    if (!out) return MOE_ERR_ARG;
    *out = nullptr;
    if (!layers || !router_w || n_layers < 1 || n_layers > moe::kStackMaxLayers) return MOE_ERR_ARG;
    const moe_ctx *l0 = layers[0];
    if (!l0) return MOE_ERR_ARG;
    for (int l = 0; l < n_layers; ++l) {
        const moe_ctx *h = layers[l];
        if (!h || h->E != l0->E || h->H != l0->H || h->I != l0->I || h->k != l0->k) return MOE_ERR_ARG;
        if (!h->loaded) return MOE_ERR_NOT_LOADED;
        // the stack kernel reads MXFP4 or NVFP4 experts, one format per stack
        if (h->s8 || h->nv != l0->nv) return MOE_ERR_ARG;
        if (h->device != l0->device) return MOE_ERR_NOT_DEVICE;
    }
    int dev = -1, sms = 0;
    int rc = current_device_ok(&dev, &sms);
    if (rc != MOE_OK) return rc;
    if (dev != l0->device) return MOE_ERR_NOT_DEVICE;
    moe::StackPlan plan;
    if (!moe::stack_plan(l0->E, l0->H, l0->I, l0->k, sms, &plan, l0->nv)) return MOE_ERR_ARG;
    for (int l = 0; l < n_layers; ++l) {
        if ((rc = check_device_ptr(l0, router_w[l], 16)) != MOE_OK) return rc;
        if (router_bias && router_bias[l] && (rc = check_device_ptr(l0, router_bias[l], 4)) != MOE_OK)
            return rc;
    }
    moe_stack_ctx *s = new (std::nothrow) moe_stack_ctx;
    if (!s) return MOE_ERR_ARG;
    s->L = n_layers;
    s->E = l0->E;
    s->H = l0->H;
    s->I = l0->I;
    s->k = l0->k;
    s->nv = l0->nv;
    s->device = dev;
    s->num_sms = sms;
    s->plan = plan;
    for (int l = 0; l < n_layers; ++l) {
        const moe_ctx *h = layers[l];
        moe::StackLayer &ly = s->layer[l];
        ly.codes_base = h->codes_base;
        ly.scales_base = h->scales_base;
        ly.table = h->d_table;
        ly.router_w = router_w[l];
        ly.bias = router_bias ? router_bias[l] : nullptr;
        ly.gscale = h->gscale;
    }
    *out = s;
    return MOE_OK;
}

int moe_stack_destroy(moe_stack_t s) {
    delete s;
    return MOE_OK;
}

int moe_stack_workspace_bytes(moe_stack_t s, size_t *bytes) {
    if (!s || !bytes) return MOE_ERR_ARG;
    *bytes = stack_ws_layout(s).total;
    return MOE_OK;
}

int moe_stack_set_workspace(moe_stack_t s, void *workspace, size_t bytes) {
    if (!s || !workspace) return MOE_ERR_ARG;
    int rc;
    moe_ctx probe;
    probe.device = s->device;
    if ((rc = check_device_ptr(&probe, workspace, 256)) != MOE_OK) return rc;
    if (bytes < stack_ws_layout(s).total) return MOE_ERR_WORKSPACE;
    if ((rc = cuda_rc(cudaMemset(workspace, 0, bytes))) != MOE_OK) return rc;
    s->ws = static_cast<uint8_t *>(workspace);
    s->ws_bytes = bytes;
    return MOE_OK;
}

int moe_stack_set_spin_limit(moe_stack_t s, int polls) {
    if (!s || polls < 0) return MOE_ERR_ARG;
    s->spin_limit = polls;
    return MOE_OK;
}

int moe_stack_set_trace(moe_stack_t s, unsigned long long *trace, size_t bytes) {
    if (!s) return MOE_ERR_ARG;
    if (!trace) {
        s->trace = nullptr;
        return MOE_OK;
    }
    const size_t need = (size_t)s->L * s->num_sms * moe::kStackTraceSlots * sizeof(unsigned long long);
    if (bytes < need) return MOE_ERR_WORKSPACE;
    moe_ctx probe;
    probe.device = s->device;
    int rc;
    if ((rc = check_device_ptr(&probe, trace, 8)) != MOE_OK) return rc;
    s->trace = trace;
    return MOE_OK;
}

int moe_stack_decode(moe_stack_t s, uint16_t *r, uint16_t *r_hist, uint16_t *xn_hist,
                     float *logits, int32_t *topk_ids, float *topk_w, void *stream) {
    if (!s) return MOE_ERR_ARG;
    if (!s->ws) return MOE_ERR_NOT_LOADED;
    moe_ctx probe;
    probe.device = s->device;
    int rc;
    if ((rc = check_device_ptr(&probe, r, 16)) != MOE_OK) return rc;
    if (r_hist && (rc = check_device_ptr(&probe, r_hist, 16)) != MOE_OK) return rc;
    if (xn_hist && (rc = check_device_ptr(&probe, xn_hist, 16)) != MOE_OK) return rc;
    if (logits && (rc = check_device_ptr(&probe, logits, 4)) != MOE_OK) return rc;
    if (topk_ids && (rc = check_device_ptr(&probe, topk_ids, 4)) != MOE_OK) return rc;
    if (topk_w && (rc = check_device_ptr(&probe, topk_w, 4)) != MOE_OK) return rc;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev != s->device) return MOE_ERR_NOT_DEVICE;
    const StackWs W = stack_ws_layout(s);
    moe::StackParams p;
    memset(&p, 0, sizeof p);
    p.L = s->L;
    p.E = s->E;
    p.H = s->H;
    p.I = s->I;
    p.k = s->k;
    p.nv = s->nv;
    p.codes_stride = (size_t)s->I * s->H / 2;
    p.scales_stride = (size_t)s->I * s->H / (s->nv ? 16 : 32);
    p.r = r;
    p.r_hist = r_hist;
    p.xn_hist = xn_hist;
    p.logits_hist = logits;
    p.ids_hist = topk_ids;
    p.w_hist = topk_w;
    p.x_tag = reinterpret_cast<uint2 *>(s->ws + W.x_tag);
    p.lg_tag = reinterpret_cast<uint2 *>(s->ws + W.lg_tag);
    p.h_tag = reinterpret_cast<uint2 *>(s->ws + W.h_tag);
    p.seq = reinterpret_cast<unsigned *>(s->ws + W.seq);
    p.abort = reinterpret_cast<unsigned *>(s->ws + W.abort);
    p.status = reinterpret_cast<unsigned *>(s->ws + W.status);
    p.spin_limit = s->spin_limit;
    p.trace = s->trace;
    p.plan = s->plan;
    for (int l = 0; l < s->L; ++l) p.layer[l] = s->layer[l];
    return cuda_rc(moe::launch_stack(p, s->num_sms, static_cast<cudaStream_t>(stream)));
}

int moe_stack_get_status(moe_stack_t s, void *stream, unsigned *device_status) {
    if (!s || !device_status) return MOE_ERR_ARG;
    if (!s->ws) return MOE_ERR_NOT_LOADED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StackWs W = stack_ws_layout(s);
    unsigned *d = reinterpret_cast<unsigned *>(s->ws + W.status);
    int rc;
    if ((rc = cuda_rc(cudaStreamSynchronize(st))) != MOE_OK) return rc;
    unsigned v = 0;
    if ((rc = cuda_rc(cudaMemcpyAsync(&v, d, sizeof v, cudaMemcpyDeviceToHost, st))) != MOE_OK)
        return rc;
    if ((rc = cuda_rc(cudaMemsetAsync(d, 0, sizeof v, st))) != MOE_OK) return rc;
    if ((rc = cuda_rc(cudaStreamSynchronize(st))) != MOE_OK) return rc;
    *device_status = v;
    return MOE_OK;
}

const char *moe_status_string(int status) {
    switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_ARG: return "MOE_ERR_ARG: invalid argument";
    case MOE_ERR_NOT_LOADED: return "MOE_ERR_NOT_LOADED: weights or workspace not set";
    case MOE_ERR_NOT_DEVICE: return "MOE_ERR_NOT_DEVICE: pointer is not memory of the current device";
    case MOE_ERR_ALIGN: return "MOE_ERR_ALIGN: pointer not aligned";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime error";
    case MOE_ERR_DEVICE_STATUS: return "MOE_ERR_DEVICE_STATUS: a kernel flagged invalid input";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: device is not sm_100";
    default: return "unknown moe status";
    }
}

int moe_device_check(void) { return current_device_ok(nullptr, nullptr); }

int moe_debug_dequant(const uint8_t *codes, const uint8_t *scales, int64_t n, float *out,
                      void *stream) {
    if (n < 0 || n % 32) return MOE_ERR_ARG;
    int rc = current_device_ok(nullptr, nullptr);
    if (rc != MOE_OK) return rc;
    if (n == 0) return MOE_OK;
    if ((rc = check_device_ptr(nullptr, codes, 16)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(nullptr, scales, 1)) != MOE_OK) return rc;
    if ((rc = check_device_ptr(nullptr, out, 16)) != MOE_OK) return rc;
    return cuda_rc(moe::launch_debug_dequant(codes, scales, n, out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
