// kernels.cuh — launch parameters and entry points of the sm_100a kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace moe {

// One-time host set-up per (call site, device): a kernel's dynamic
// shared-memory limit is a property of the function in the context of the
// device that is current when it is set, so a process that drives several
// GPUs must set it on each.  Thread-safe; `set` runs with the device current.
struct PerDeviceOnce {
    static constexpr int kMaxDevices = 64;
    std::atomic<unsigned long long> done{0};
    std::mutex m;
};
template <class F>
inline cudaError_t per_device_once(PerDeviceOnce &o, F &&set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long bit = 1ull << dev;
    if (o.done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    std::lock_guard<std::mutex> g(o.m);
    if (o.done.load(std::memory_order_relaxed) & bit) return cudaSuccess;
    e = set();
    if (e == cudaSuccess) o.done.fetch_or(bit, std::memory_order_release);
    return e;
}

constexpr int kDecodeMaxT = 4;      // tokens handled by the per-(token,slot) GEMV path
constexpr int kMaxTopK = 8;
constexpr int kGemvThreads = 512;   // gate/up GEMV: 16 warps, one CTA per SM
constexpr int kDownThreads = 768;   // down GEMV + combine: 24 warps, one CTA per SM
constexpr int kRouteThreads = 256;  // 8 warps, one expert row per warp
constexpr unsigned kBadExpertId = 0x1u;
constexpr size_t kMaxDecodeSmem = 200 * 1024;  // dynamic shared memory cap of the GEMVs

struct RouteParams {
    const uint16_t *x;      // [T][H] BF16 (residual stream when rmsnorm)
    const uint16_t *wr;     // [E][H] BF16
    const float *bias;      // [E] or null
    uint16_t *x_norm;       // [T][H] or null
    float *logits_ws;       // [T][E] workspace
    float *logits_out;      // [T][E] or null
    int32_t *ids;           // [T][k]
    float *w;               // [T][k]
    unsigned *counters;     // [T], zero between calls
    uint32_t *x16;          // [T][H/2] FP16-staged routed vector (f16x2 words) or null
    int *x16_exp;           // [T] its staging exponent c (values are x * 2^-c)
    int T, E, H, k;
    int rmsnorm;
    int sigmoid;            // sigmoid scoring (bias steers selection only)
    float eps;
};

struct GateUpParams {
    const ExpertPtrs *table;  // [E]
    // contiguous layout fast path (weights bound with one base address):
    // matrix m of expert e at base + (3 e + m) * stride; null: use the table
    const uint8_t *codes_base, *scales_base;
    size_t codes_stride, scales_stride;
    const uint16_t *x;        // [T][H]
    const uint32_t *x16;      // [T][H/2] pre-staged FP16 x (from the router) or null
    const int *x16_exp;       // [T] staging exponents of x16
    const int32_t *ids;       // [T][k] given routing, or null: route from logits
    const float *logits;      // [T][E] when ids is null
    int32_t *ids_out;         // [T][k] or null: written by CTA 0 when routing
    float *w_out;             // [T][k] or null: from logits
    uint16_t *h;              // [T][k][I]
    unsigned *status;
    int T, k, E, H, I;
    int prefetch_down;        // L2-prefetch the selected down matrices
    uint32_t pf_codes, pf_scales;  // per-CTA prefetch slice (bytes, multiple of 16)
    int nslots;               // shared-memory ring slots of the bulk-copy kernel
    int nv;                   // NVFP4 weights: E4M3 scale per 16 (else E8M0 per 32)
    const float *gscale;      // NVFP4: [E][2] FP32 multipliers (gate/up, down)
};

// Routing handed from the fused router + gate/up kernel to the down kernel of
// the same call, one copy per CTA index i (both grids have the same size).
// Every entry is an 8-byte word {tag, value} written and read as one access,
// so a reader that sees the expected tag also sees the value: gate/up CTA i
// writes its ids / w with tag seq[i] + 1 and then stores seq[i] + 1; down CTA
// i polls (bounded) until its entries carry ack[i] + 1, then stores that in
// ack[i].  Between calls seq[i] == ack[i].  The down kernel can thus route
// before its programmatic-launch wait without relying on that wait.
constexpr int kHandMaxCtas = 256;
constexpr int kHandStride = kDecodeMaxT * kMaxTopK;
struct RouteHandoff {
    unsigned *seq;   // [kHandMaxCtas] publications made by gate/up CTA i
    unsigned *ack;   // [kHandMaxCtas] publications taken by down CTA i
    uint2 *ent;      // [kHandMaxCtas][kHandStride][2]: {tag, id}, {tag, w bits}
};

// Router half of the fused router + gate/up launch.
constexpr int kFusedMaxE = 256;  // experts of the fused router (E/2 per CTA)
struct FusedRouteParams {
    const uint16_t *xr;      // [T][H] layer input (the residual stream when rmsnorm)
    const uint16_t *wr;      // [E][H] BF16 router
    const float *bias;       // [E] or null
    uint16_t *x_norm;        // [T][H] written when rmsnorm (CTA 0)
    float *logits_out;       // [T][E] or null
    uint2 *logit_ent;        // [T][E] {tag, logit bits}: CTA e % G publishes expert e
    RouteHandoff hand;
    int rmsnorm;
    float eps;
    unsigned region_bytes;   // dynamic shared memory before the routed-vector buffer
};

// Down half of the one-launch layer (router + gate/up + down in one grid).
struct LayerDownParams {
    const uint16_t *residual;  // [T][H] or null
    uint16_t *y;               // [T][H]
    uint2 *h_tag;              // [T][k][I] {tag, BF16 h}: h exchanged between the CTAs
    int rows_per_cta;          // R: output rows of each CTA
    unsigned down_off;         // dynamic shared memory offset of the down region
};

struct DownParams {
    const ExpertPtrs *table;
    const uint8_t *codes_base, *scales_base;  // contiguous layout fast path (or null)
    size_t codes_stride, scales_stride;
    const uint16_t *h;         // [T][k][I]
    const int32_t *ids;        // [T][k] given routing, or null: route from logits
    const float *w;            // [T][k] given routing weights (ids != null)
    const float *logits;       // [T][E] when ids is null
    const uint16_t *residual;  // [T][H] or null
    uint16_t *y;               // [T][H]
    uint16_t *o_keep;          // [T][k][H] or null
    unsigned *status;
    int T, k, E, H, I;
    int rows_per_cta;
    RouteHandoff hand;         // used when ids and logits are both null
    int nv;                    // NVFP4 weights (see GateUpParams)
    const float *gscale;       // NVFP4: [E][2] FP32 multipliers
};

// The (token, expert)-sorted grouped path (grouped.cu), for batches of tokens.
constexpr int kGroupedMaxT = 2048;  // tokens per grouped launch sequence (more: chunks)
// Tensor maps of a handle's packed codes for the tcgen05 products (one per
// matrix kind: 0 gate/up, 1 down), encoded when first needed and again only
// when the bound weights change; opaque CUtensorMap bytes.  Owned by the
// handle (calls on one handle are serialised by its owner).
struct TcMapCache {
    alignas(64) unsigned char map[2][128];
    const uint8_t *base[2] = {nullptr, nullptr};
    int E[2] = {0, 0}, rows[2] = {0, 0}, K[2] = {0, 0};
};

struct GroupedParams {
    const ExpertPtrs *table;
    const uint8_t *codes_base, *scales_base;  // contiguous layout fast path (or null)
    size_t codes_stride, scales_stride;
    const uint16_t *x;         // [T][H] BF16
    const int32_t *ids;        // [T][k]
    const float *w;            // [T][k]
    const uint16_t *residual;  // [T][H] or null
    uint16_t *y;               // [T][H]
    uint16_t *o_keep;          // [T][k][H] or null
    // workspace
    int *perm;                 // [T k] pair indices t k + j, sorted by (expert, pair)
    int *offs;                 // [E + 1] start of each expert's segment in perm
    uint32_t *x16;             // [T][H/2] FP16-staged x (f16x2 words)
    int *x_exp;                // [T] staging exponents of x16
    uint16_t *h;               // [T k][I] BF16 SwiGLU outputs
    uint32_t *h16;             // [T k][I/2] FP16-staged h
    int *h_exp;                // [T k] staging exponents of h16
    uint16_t *o;               // [T k][H] BF16 expert outputs
    unsigned *status;
    int T, k, E, H, I;
    int tcgen05;               // products on tcgen05 (else mma.sync tiles)
    int nv;                    // NVFP4 weights: E4M3 scale per 16 (mma.sync tiles only)
    int s8;                    // sym8 weights: int8, binary16 scale per 32 (mma.sync tiles only)
    const float *gscale;       // NVFP4: [E][2] FP32 multipliers (gate/up, down)
    TcMapCache *tc_maps;       // the handle's tensor-map cache (host), or null
};
bool grouped_supported(int E, int H, int I, int nv = 0, int s8 = 0);
cudaError_t launch_grouped(const GroupedParams &p, cudaStream_t s, bool pdl);
// Products on tcgen05 (grouped_tc.cu): chosen by the forward when the groups
// average at least kTcAutoGroup pairs (the mma.sync tiles convert the codes
// again for every 8 tokens, the tcgen05 CTAs once per 128), or on request.
constexpr int kTcAutoGroup = 40;
bool grouped_tc_supported(int H, int I, int nv = 0);
cudaError_t launch_grouped_tc_gateup(const GroupedParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_grouped_tc_down(const GroupedParams &p, cudaStream_t s, bool pdl);

// Host-side launchers (decode.cu).  `pdl` sets programmatic stream
// serialization so the kernel may start while the previous one drains.
cudaError_t launch_route(const RouteParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_route_logits(const RouteParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_topk(const RouteParams &p, cudaStream_t s, bool pdl);
bool gateup_tma_supported(int H);
int gateup_tma_slots(int H, int nv = 0);
cudaError_t launch_gateup_decode(const GateUpParams &p, int grid, cudaStream_t s, bool pdl);
cudaError_t launch_down_decode(const DownParams &p, int grid, cudaStream_t s, bool pdl);
// Fused router + gate/up (layer.cu): one CTA per SM, grid = SM count.  layer_gateup_plan returns the dynamic shared memory and
// ring slots for (T, E, H), or false when the shape needs the unfused path.
bool layer_gateup_plan(int T, int E, int H, int grid, size_t *smem, int *nslots,
                       unsigned *region_bytes);
cudaError_t launch_layer_gateup(const GateUpParams &p, const FusedRouteParams &r, int grid,
                                size_t smem, cudaStream_t s, bool pdl);
// The whole layer in one launch (T small enough for the gate/up ring, the
// routed vector and the CTA's down rows to share one SM's shared memory, and
// I a multiple of 512): layer_plan returns its dynamic shared memory, ring
// slots and the offsets, or false.
bool layer_plan(int T, int E, int H, int I, int k, int grid, size_t *smem, int *nslots,
                unsigned *region_bytes, unsigned *down_off, int *rows_per_cta);
cudaError_t launch_layer(const GateUpParams &p, const FusedRouteParams &r,
                         const LayerDownParams &d, int grid, size_t smem, cudaStream_t s,
                         bool pdl);
// ------------------------------------------------------------------------
// The whole batch-1 decode step of a stack of layers in one persistent,
// cooperative launch (stack.cu): one CTA per SM, every layer's RMSNorm,
// router, top-k, gate/up + SwiGLU, down, combine and residual add, with the
// three grid-wide hand-offs of a layer (layer input, router logits, h) done
// through tagged 8-byte words {tag, value} in the workspace.
constexpr int kStackMaxLayers = 64;
constexpr int kStackThreads = 512;  // 16 warps: 128 registers per thread
constexpr int kStackTraceSlots = 16;  // phase time stamps per layer and CTA (profiling)
// Exchange layout of the stack kernel's tagged words: word w of an exchange
// buffer sits at uint2 index (w / 4) * kStkLineWords + w % 4, i.e. each
// 4-word piece (and each router logit, at index e * kStkLineWords) on a
// 128-byte line of its own.  Every CTA polls every line of an exchange, so
// packed words would put ~150 readers' polls on a few L2 lines; spread, the
// polls of one round go to as many lines as there are pieces (measured: a
// grid-wide exchange of 1,036 words took 2.5 us packed, 1.5 us spread).
constexpr size_t kStkLine = 128;
constexpr int kStkLineWords = (int)(kStkLine / 8);

struct StackLayer {
    const uint8_t *codes_base, *scales_base;  // contiguous [E][3][...], or null
    const ExpertPtrs *table;                  // device expert table (codes_base null)
    const uint16_t *router_w;                 // [E][H] BF16
    const float *bias;                        // [E] or null
    const float *gscale;                      // NVFP4: [E][2] FP32 multipliers (gate/up, down)
};

// Shared-memory plan of the stack kernel (host-computed, passed by value).
struct StackPlan {
    size_t smem;                         // dynamic shared memory bytes
    unsigned off_gu, off_dn, off_rt, off_sx, off_x16, off_sh, off_so;
    int np_max;   // gate/up row pairs of the largest CTA share
    int ppc;      // row pairs per code piece
    int R;        // down rows of the largest CTA share (a multiple of U)
    int U;        // down rows per unit of the CTA split (2 or 4: 16-byte scale copies)
};

struct StackParams {
    int L, E, H, I, k;
    int nv;                               // NVFP4 layers (E4M3 scale per 16) else MXFP4
    size_t codes_stride, scales_stride;   // bytes per matrix (contiguous layers)
    uint16_t *r;                          // [H] residual stream, in and out
    uint16_t *r_hist;                     // [L][H] each layer's input, or null
    uint16_t *xn_hist;                    // [L][H] each layer's routed vector, or null
    float *logits_hist;                   // [L][E] or null
    int32_t *ids_hist;                    // [L][k] or null
    float *w_hist;                        // [L][k] or null
    // workspace
    // exchange buffers, words spread one piece per line (kStkLineWords)
    uint2 *x_tag;                         // [H/2] {tag, 2 x BF16} layer outputs
    uint2 *lg_tag;                        // [E] {tag, FP32} router logits
    uint2 *h_tag;                         // [k][I/2] {tag, 2 x BF16} SwiGLU outputs
    unsigned *seq;                        // [grid] launches made by CTA b
    unsigned *abort;                      // launch tag of a launch that gave up
    unsigned *status;                     // device status bits
    int spin_limit;                       // polls of a tagged-word wait before it gives up
    unsigned long long *trace;            // [L][grid][kStackTraceSlots] time stamps, or null
    StackPlan plan;
    StackLayer layer[kStackMaxLayers];
};

// False when the shape is outside what the stack kernel holds (then the
// layers run one by one).  nv: NVFP4 layers (twice the scale bytes).
bool stack_plan(int E, int H, int I, int k, int grid, StackPlan *plan, int nv = 0);
cudaError_t launch_stack(const StackParams &p, int grid, cudaStream_t s);

cudaError_t launch_debug_dequant(const uint8_t *codes, const uint8_t *scales, int64_t n,
                                 float *out, cudaStream_t s);
size_t gateup_decode_smem(int T, int H);
size_t down_decode_smem(int T, int k, int I, int rows_per_cta);
constexpr size_t kDownSmemMax = 200 * 1024;
bool decode_shape_supported(int H, int I);

// ---- sym8 experts (int8 weights, binary16 scale per 32; sym8.cu) ----
constexpr int kS8MaxT = 4;                // tokens per launch pair
constexpr size_t kS8SmemMax = 48 * 1024;  // staged x / h per CTA
struct Sym8Params {
    const ExpertPtrs *table;     // [E]: codes [3][rows][K] int8, scales [3][rows][K/32] binary16
    const uint16_t *x;           // [T][H] BF16
    const int32_t *ids;          // [T][k] given routing, or null: route from logits
    const float *w;              // [T][k]
    const float *logits;         // [T][E] router logits when ids is null (softmax top-k)
    int32_t *ids_out;            // [T][k] or null: written by gate/up CTA 0 when routing
    float *w_out;                // [T][k] or null
    const uint16_t *residual;    // [T][H] or null
    uint16_t *y;                 // [T][H]
    uint16_t *h;                 // [T][k][I] BF16 SwiGLU outputs (workspace)
    uint16_t *o_keep;            // [T][k][H] expert outputs, or null
    unsigned *status;
    int T, E, H, I, k;
};
bool sym8_supported(int H, int I, int k);
int sym8_max_chunk(int H, int I, int k);
cudaError_t launch_sym8(const Sym8Params &p, int num_sms, bool run_gu, bool run_dn,
                        cudaStream_t s, bool pdl);

}  // namespace moe
