/*
 * moe_mxfp4.h — C ABI of the packed-MXFP4 W4A16 top-4 MoE expert FFN for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference"):
 *   - table "Model and quantization": expert weights are E2M1 FP4 values,
 *     two per byte, with one E8M0 scale per 32 values; activations are BF16;
 *     the packed GEMVs accumulate in FP32 and produce BF16 outputs; each MoE
 *     layer routes every token to 4 of its experts.
 *   - section "GPU routing inside resident-layer graphs": router projection,
 *     expert bias where configured, dynamic top-k selection and routing
 *     coefficients, recomputed on the GPU each call, with no copy of the
 *     selected ids to the host.
 *   - section "What was optimized" > "Grouped top-4 expert execution": one
 *     grouped packed GEMV for gate, one for up, activation and
 *     multiplication, one grouped packed GEMV for down, and a fused
 *     routing-weighted combination that keeps the sequential BF16
 *     multiply/add rounding of a one-expert-at-a-time runner.
 *   - section "Direct reads from GPU-resident weights": experts are read in
 *     place through a persistent device table of expert addresses; no
 *     staging copy, no BF16 copy of the weights.
 * The SwiGLU expert is three matrices, gate and up (I x H) and down (H x I)
 * ("LFM2.5-24B-A2B on Your Own Hardware", section "Where do the 2.45B active
 * parameters actually go?").
 *
 * Exact arithmetic of one (token t, slot j) with expert e = ids[t][j]:
 *   g = BF16(sum_h Wg[e][i][h] x[t][h])       (FP32 accumulation)
 *   u = BF16(sum_h Wu[e][i][h] x[t][h])
 *   h[i] = BF16( BF16(silu(g)) * u )
 *   o[n] = BF16(sum_i Wd[e][n][i] h[i])
 * and the combine, in slot order j = 0..k-1, starting from y = +0:
 *   y = BF16( y + BF16( o_j * BF16(w_j) ) )
 *   optionally followed by y = BF16(residual + y).
 *
 * Conventions for every call:
 *   - BF16 tensors are passed as uint16_t bit patterns.
 *   - All tensors are row-major and contiguous.  Pointers documented as
 *     "device" must point to memory of the current CUDA device (cudaMalloc'd,
 *     e.g. by PyTorch); the library checks this and returns
 *     MOE_ERR_NOT_DEVICE otherwise.  Device pointers must be 16-byte aligned
 *     (MOE_ERR_ALIGN otherwise).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 *     moe_route / moe_forward only enqueue kernels: they never allocate,
 *     never synchronise and never copy weights, so they may be captured in a
 *     CUDA graph.
 *   - The library never takes ownership of caller memory: weights, workspace
 *     and I/O buffers must stay valid until moe_destroy (weights, workspace)
 *     or until the enqueued work completes (inputs/outputs).
 *   - Every call returns a moe_status_t; nothing is thrown across the ABI.
 *     A call that returns an error has enqueued nothing.
 *
 * Packed weight layout (the model card calls the checkpoint layout "custom"
 * and does not describe it; this is the layout of this library):
 *   codes  uint8 [E][3][rows][K/2]: matrix 0 = gate (rows I, K H),
 *          1 = up (rows I, K H), 2 = down (rows H, K I).  Element 2i of a
 *          row is the low nibble of byte i, element 2i+1 the high nibble.
 *          E2M1 code c: sign = bit 3, magnitude {0,.5,1,1.5,2,3,4,6}[c&7].
 *   scales uint8 [E][3][rows][K/32]: E8M0, value 2^(s-127), s = 255 is NaN;
 *          one per 32 consecutive K elements.
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_ctx *moe_handle_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_ARG = -1,           /* bad shape, null pointer, T out of range  */
    MOE_ERR_NOT_LOADED = -2,    /* weights or workspace not set yet         */
    MOE_ERR_NOT_DEVICE = -3,    /* pointer is not memory of this device     */
    MOE_ERR_ALIGN = -4,         /* pointer not 16-byte aligned              */
    MOE_ERR_WORKSPACE = -5,     /* workspace too small for this T           */
    MOE_ERR_CUDA = -6,          /* a CUDA runtime call failed               */
    MOE_ERR_DEVICE_STATUS = -7, /* a kernel flagged bad input (ids)         */
    MOE_ERR_UNSUPPORTED = -8    /* current device is not sm_100             */
} moe_status_t;

/* Bits of the device status word read by moe_get_status. */
#define MOE_DEVICE_BAD_EXPERT_ID 0x1u /* an id outside [0, E): slot zeroed */
#define MOE_DEVICE_TIMEOUT 0x2u       /* a bounded in-kernel wait gave up;
                                         outputs of that call are invalid */

/* Flags of moe_route_ex. */
#define MOE_ROUTE_RMSNORM 0x1u /* x is a residual stream r: route
                                  xn = BF16(r / sqrt(mean(r^2) + 1e-6))
                                  and write xn to x_norm */
#define MOE_ROUTE_SIGMOID 0x2u /* sigmoid scoring: s_e = sigmoid(l_e) of
                                  the unbiased logit; the k experts with
                                  the largest s_e + bias_e are selected
                                  (bias only steers selection); their
                                  coefficients are s_j / sum of the k
                                  selected s.  Without it: top-k of the
                                  (biased) logits, softmax over them.  */

/* Flags of moe_forward_ex. */
#define MOE_FWD_KEEP_INTERMEDIATES 0x1u /* also store h [T][k][I] and
                                           o [T][k][H] in the workspace
                                           (moe_get_intermediates)         */
#define MOE_FWD_FORCE_DECODE 0x2u  /* per-(token,slot) GEMV path            */
#define MOE_FWD_FORCE_GROUPED 0x4u /* (token,expert)-sorted grouped path    */
#define MOE_FWD_PHASE_GATEUP 0x8u  /* run only the gate/up/SwiGLU kernel(s);
                                      h stays in the workspace              */
#define MOE_FWD_PHASE_DOWN 0x10u   /* run only the down + combine kernel(s)
                                      on the h of the preceding
                                      MOE_FWD_PHASE_GATEUP call (same T,
                                      ids, same handle and workspace); the
                                      two calls together equal one forward  */
#define MOE_FWD_FORCE_TCGEN05 0x20u /* grouped path with its products on
                                      tcgen05 (TMEM accumulators, TMA tensor
                                      loads of the packed codes); needs the
                                      contiguous weights of moe_load_packed
                                      or moe_load_packed_nvfp4 and H, I
                                      multiples of 128, else ARG           */
#define MOE_FWD_FORCE_MMA 0x40u    /* grouped path with its products on
                                      mma.sync tiles (never tcgen05)        */

/* Create a layer of E experts with hidden size H, intermediate size I and
 * top_k experts per token.  Requires H % 32 == 0, I % 32 == 0,
 * 32 <= H <= 4096, 32 <= I <= 4096, 1 <= top_k <= min(E, 8), E <= 1024.  Host-only: allocates the
 * handle, touches no GPU.  *out receives the handle (NULL on error).
 * Errors: MOE_ERR_ARG. */
MOE_API int moe_create(int E, int H, int I, int top_k, moe_handle_t *out);

/* Release the handle and the small device block it allocated at load time
 * (expert table, status word).  Caller memory is never freed.  NULL is a
 * no-op.  Synchronises the device if a device block exists. */
MOE_API int moe_destroy(moe_handle_t h);

/* Bind contiguously stored packed weights (layout above): codes device
 * uint8 [E][3][I*H/2], scales device uint8 [E][3][I*H/32].  Both 16-byte
 * aligned.  Nothing is copied: the library builds the device expert table
 * from these base addresses and reads the weights in place.  Allocates the
 * handle's device block (expert table + status word) on first use and
 * synchronises the device once.  Errors: ARG, NOT_DEVICE, ALIGN, CUDA,
 * UNSUPPORTED. */
MOE_API int moe_load_packed(moe_handle_t h, const uint8_t *codes_u8,
                    const uint8_t *scales_e8m0);

/* Bind experts stored anywhere: codes_ptrs / scales_ptrs are HOST arrays of
 * 3*E DEVICE pointers, entry 3*e+m pointing at matrix m (0 gate, 1 up,
 * 2 down) of expert e in the per-matrix layout above ([rows][K/2] and
 * [rows][K/32]).  Every pointer 16-byte aligned.  Same ownership and
 * errors as moe_load_packed. */
MOE_API int moe_load_expert_table(moe_handle_t h, const uint8_t *const *codes_ptrs,
                          const uint8_t *const *scales_ptrs);

/* Bind contiguously stored NVFP4 experts (page "primitive-ai/LFM2.5-24B-
 * A2B-NVFP4A16", section "What's quantized to what": NVFP4 routed experts,
 * 16-bit compute, w1 and w3 of an expert sharing one global scale).
 * codes: device uint8 [E][3][I*H/2], E2M1 packed as for MXFP4; scales_e4m3:
 * device uint8 [E][3][I*H/16], one FP8 E4M3 scale per 16 consecutive K
 * elements; global_scales: device FP32 [E][2], per expert the multiplier of
 * gate and up, then that of down.  Weight = e2m1(code) * e4m3(scale) *
 * multiplier.  codes / scales 16-byte aligned, global_scales 4-byte aligned;
 * read in place, caller-owned.  Requires H a multiple of 512 up to 4096 (the
 * bulk-copy gate/up kernel).  NVFP4 layers run the per-(token, slot) path
 * for T = 1..4 and the grouped path beyond: mma.sync products (each 16-
 * element block's partial product scaled by its E4M3 scale in FP32, the
 * multiplier applied with the activation staging scale), or, for large
 * groups, tcgen05 products (A = code x its block's E4M3 scale in BF16,
 * exact; the multiplier applied to the FP32 accumulator).  The one-launch stack
 * takes NVFP4 layers; no fused launch structures.  moe_load_packed /
 * moe_load_expert_table switch the handle back to MXFP4.  Errors: as
 * moe_load_packed. */
MOE_API int moe_load_packed_nvfp4(moe_handle_t h, const uint8_t *codes_u8,
                                  const uint8_t *scales_e4m3, const float *global_scales);

/* Bind contiguously stored sym8 experts (page "LFM2.5-8B-A1B — Core AI
 * (.aimodel)", table "Provenance", row "Weight format": symmetric-linear int8
 * weights with one scale per K-block of 32).  codes_s8: device int8
 * [E][3][I*H], row-major rows of K weights per matrix (gate, up: I rows of H;
 * down: H rows of I), one two's-complement byte per weight; scales_f16:
 * device uint16 [E][3][I*H/32], one IEEE binary16 scale (little-endian bit
 * pattern) per 32 consecutive K elements of a row.  Weight = q * scale, no
 * zero point.  codes 16-byte aligned, scales 2-byte aligned; read in place
 * through the handle's device pointer table, caller-owned.  Requires H and I
 * multiples of 32 with one token's H (gate/up) and k*I (down) BF16 values
 * within 48 KB.  sym8 layers run the per-(token, slot) GEMVs (FP32 products
 * and sums) up to 4 tokens, and beyond that (or with FORCE_GROUPED /
 * FORCE_MMA) the grouped mma.sync products: int8 rows converted to FP16
 * exactly, the binary16 scale applied per 32-element group in FP32.  The
 * grouped products need the scales 4-byte aligned and H, I multiples of 128
 * within the tiles' shared memory (H, I <= 4096 and both products' tiles
 * within 220 KB); otherwise every T runs the GEMVs in chunks of up to 4
 * tokens (FORCE_GROUPED / FORCE_MMA then return ARG).  No tcgen05 products
 * (FORCE_TCGEN05 returns ARG), no fused launch structures, no stack kernel.
 * moe_load_packed,
 * moe_load_packed_nvfp4 and moe_load_expert_table switch the handle to their
 * format.  Errors: ARG (null pointer, unsupported shape), NOT_DEVICE, CUDA. */
MOE_API int moe_load_packed_sym8(moe_handle_t h, const int8_t *codes_s8,
                                 const uint16_t *scales_f16);

/* Bytes of device workspace needed for up to max_tokens tokens per call.
 * Errors: ARG. */
MOE_API int moe_workspace_bytes(moe_handle_t h, int max_tokens, size_t *bytes);

/* Give the handle a device workspace (owned by the caller, 256-byte
 * aligned, at least moe_workspace_bytes(max_tokens) bytes).  Zeroes it
 * (synchronously).  Several handles may share one workspace if their calls
 * are ordered on one stream.  Errors: ARG, NOT_DEVICE, ALIGN, WORKSPACE,
 * CUDA. */
MOE_API int moe_set_workspace(moe_handle_t h, void *workspace, size_t bytes,
                      int max_tokens);

/* Routing for T tokens (1 <= T <= max_tokens of the workspace):
 *   logits[t][e] = sum_h x[t][h] * router_w[e][h]   (FP32 accumulation)
 *                  (+ router_bias[e] if router_bias != NULL)
 *   topk_ids[t][0..k-1] = experts of the k largest logits, descending,
 *                          equal logits -> lower expert id first
 *   topk_w[t][j] = softmax over the k selected logits (FP32).
 * x: device BF16 [T][H]; router_w: device BF16 [E][H]; router_bias: device
 * FP32 [E] or NULL; topk_ids: device int32 [T][k]; topk_w: device FP32
 * [T][k].  Errors: ARG, NOT_LOADED (no workspace), NOT_DEVICE, ALIGN,
 * WORKSPACE, CUDA. */
MOE_API int moe_route(moe_handle_t h, const uint16_t *x, int T,
              const uint16_t *router_w, const float *router_bias,
              int32_t *topk_ids, float *topk_w, void *stream);

/* moe_route plus options.  flags: MOE_ROUTE_RMSNORM (then x_norm, device
 * BF16 [T][H], receives the normalised input that is routed; otherwise
 * x_norm must be NULL) and MOE_ROUTE_SIGMOID (the scoring above).  logits:
 * device FP32 [T][E] that receives the logits, or NULL: biased with the
 * softmax scoring, unbiased with MOE_ROUTE_SIGMOID (the bias enters only the
 * selection key). */
MOE_API int moe_route_ex(moe_handle_t h, const uint16_t *x, int T,
                 const uint16_t *router_w, const float *router_bias,
                 unsigned flags, uint16_t *x_norm, float *logits,
                 int32_t *topk_ids, float *topk_w, void *stream);

/* Expert FFN + combine for T tokens with given routing (e.g. from
 * moe_route):  y[t] = sequential BF16 combine of the k expert outputs.
 * x: device BF16 [T][H]; topk_ids: device int32 [T][k]; topk_w: device FP32
 * [T][k]; y: device BF16 [T][H] (must not alias x).  An id outside [0, E)
 * makes that slot contribute 0 and sets MOE_DEVICE_BAD_EXPERT_ID in the
 * device status word.  T = 1..4 runs the per-(token, slot) GEMV path;
 * larger T the (token, expert)-sorted grouped path, in chunks of up to 2048
 * tokens: its products run
 * on mma.sync tiles, or on tcgen05 (BF16 weight tiles dequantised once per
 * CTA, FP32 accumulators in tensor memory, packed codes brought in by TMA
 * tensor loads) when a chunk's groups average at least 40 (token, slot)
 * pairs per expert (T k >= 40 E) and the weights allow it (contiguous MXFP4
 * or NVFP4 from moe_load_packed / moe_load_packed_nvfp4, H and I multiples
 * of 128; sym8 weights always take the mma.sync tiles);
 * MOE_FWD_FORCE_TCGEN05 / MOE_FWD_FORCE_MMA pin the choice.  Errors: ARG,
 * NOT_LOADED, NOT_DEVICE, ALIGN, WORKSPACE, CUDA. */
MOE_API int moe_forward(moe_handle_t h, const uint16_t *x, int T,
                const int32_t *topk_ids, const float *topk_w, uint16_t *y,
                void *stream);

/* moe_forward plus options.  residual: device BF16 [T][H] or NULL; if given,
 * y = BF16(residual + combine) (residual may alias y).  flags: the
 * MOE_FWD_* bits above. */
MOE_API int moe_forward_ex(moe_handle_t h, const uint16_t *x, int T,
                   const int32_t *topk_ids, const float *topk_w,
                   const uint16_t *residual, uint16_t *y, unsigned flags,
                   void *stream);

/* One whole layer: routing + expert FFN + combine, with the routing computed
 * inside the expert kernels (no separate top-k launch, no id round trip; see
 * moe_set_fusion):
 *   - route_flags MOE_ROUTE_RMSNORM: x is a residual stream r; the layer
 *     routes and runs the experts on xn = BF16(r / sqrt(mean(r^2) + 1e-6)),
 *     written to x_norm (device BF16 [T][H], distinct from x and y).
 *   - route_flags MOE_ROUTE_SIGMOID: sigmoid scoring as in moe_route_ex.
 *   - logits (device FP32 [T][E] or NULL) receives the logits as in
 *     moe_route_ex; topk_ids / topk_w (device [T][k] or NULL) receive the
 *     routing.
 *   - residual (or NULL; may alias y and x) is added as in moe_forward_ex;
 *     fwd_flags may hold MOE_FWD_KEEP_INTERMEDIATES.
 * Results equal moe_route_ex followed by moe_forward_ex.  For T > 4, and
 * with MOE_ROUTE_SIGMOID, the call runs exactly that sequence and then
 * topk_ids / topk_w are required.
 * Errors: as moe_route_ex and moe_forward_ex. */
MOE_API int moe_layer_ex(moe_handle_t h, const uint16_t *x, int T,
                         const uint16_t *router_w, const float *router_bias,
                         unsigned route_flags, uint16_t *x_norm, float *logits,
                         int32_t *topk_ids, float *topk_w,
                         const uint16_t *residual, uint16_t *y,
                         unsigned fwd_flags, void *stream);

/* Device pointers to the intermediates kept by the last moe_forward_ex with
 * MOE_FWD_KEEP_INTERMEDIATES: h BF16 [T][k][I] (SwiGLU outputs) and o BF16
 * [T][k][H] (expert outputs before the combine).  They live in the
 * workspace until the next forward.  Errors: NOT_LOADED. */
MOE_API int moe_get_intermediates(moe_handle_t h, const uint16_t **h_out,
                          const uint16_t **o_out);

/* Synchronise the device, return the device status word (MOE_DEVICE_* bits)
 * of this handle in *device_status and clear it.  Errors: NOT_LOADED, CUDA.
 */
MOE_API int moe_get_status(moe_handle_t h, unsigned *device_status);

/* Device status of the handle's work queued on `stream` (the handle's
 * kernels must have been enqueued on that stream), then cleared: waits for
 * that stream only (moe_get_status waits for the whole device).  stream: a
 * cudaStream_t, or NULL for the legacy default stream.  The read goes to
 * pageable host memory, so it completes before the call returns.  Errors:
 * ARG, NOT_LOADED, CUDA. */
MOE_API int moe_get_status_stream(moe_handle_t h, void *stream, unsigned *device_status);

/* Packed bytes of one expert: 3*I*H/2 code bytes + 3*I*H/32 scale bytes
 * (5,013,504 for H=2048, I=1536).  Errors: ARG. */
MOE_API int moe_bytes_per_expert(moe_handle_t h, size_t *bytes);

/* Performance switches (both on by default; results do not depend on them):
 * use_pdl: launch each kernel with programmatic stream serialization so it
 * can start while the previous kernel of the stream drains; prefetch_down:
 * the gate/up kernel asks L2 to fetch the selected experts' down matrices
 * while it streams gate/up.  Errors: ARG. */
MOE_API int moe_set_tuning(moe_handle_t h, int use_pdl, int prefetch_down);

/* Launch structure of moe_layer_ex for T <= 4; results are bit-identical
 * in every mode:
 *   MOE_FUSION_NONE (default): a router launch, the gate/up launch, the down
 *     launch;
 *   MOE_FUSION_ROUTER: the RMSNorm, the router logits and the top-k run
 *     inside the gate/up launch (one CTA per SM; the CTA of index e
 *     publishes expert e's logit to the others through the workspace), and
 *     the routing reaches the down launch through the workspace;
 *   MOE_FUSION_LAYER: the whole layer in one launch (the down phase waits,
 *     bounded, for every CTA's gate/up through per-CTA words in the
 *     workspace).
 * A mode falls back to the next simpler one for shapes it cannot hold in
 * shared memory (LAYER: H <= 2048, I a multiple of 512 and small T; ROUTER:
 * E <= 256, H a multiple of 512 up to 4096) and LAYER also when
 * MOE_FWD_KEEP_INTERMEDIATES is asked.  The workspace carries per-call
 * counters for the fused modes: one workspace must not serve two calls at
 * the same time.  Errors: ARG (unknown mode). */
#define MOE_FUSION_NONE 0
#define MOE_FUSION_ROUTER 1
#define MOE_FUSION_LAYER 2
MOE_API int moe_set_fusion(moe_handle_t h, int mode);

/* ---------------------------------------------------------------------
 * A decode stack: the batch-1 decode step of n_layers MoE layers on a
 * residual stream r, in ONE kernel launch (model card sections "Grouped
 * top-4 expert execution", "GPU routing inside resident-layer graphs",
 * "Direct reads from GPU-resident weights"; the RMS cells of "CUDA Graph
 * lifetime and state management").  For each layer l in order:
 *   xn = BF16(r / sqrt(mean(r^2) + 1e-6))            (weightless RMSNorm)
 *   routing of xn as moe_route (softmax over the top-k biased logits)
 *   r  = BF16(r + combine(experts(xn)))              (as moe_forward_ex
 *                                                     with residual r)
 * i.e. exactly moe_layer_ex(MOE_ROUTE_RMSNORM, residual = y = r) per layer,
 * bit for bit.  One CTA per SM stays resident for the whole step
 * (cooperative launch) and the CTAs hand each layer's grid-wide steps to one
 * another through tagged words in the stack's workspace; every wait is
 * bounded and a wait that gives up sets MOE_DEVICE_TIMEOUT. */
typedef struct moe_stack_ctx *moe_stack_t;

/* Create a stack over n_layers (1..64) layer handles that are already bound
 * to MXFP4 weights (moe_load_packed or moe_load_expert_table), or all to
 * NVFP4 weights (moe_load_packed_nvfp4), on the current device and share E,
 * H, I, top_k.  router_w: HOST array of n_layers device
 * pointers, BF16 [E][H] each (16-byte aligned); router_bias: NULL or a HOST
 * array of n_layers device pointers, FP32 [E] or NULL each.  The layers'
 * weight bindings and these pointers are read now: rebinding a layer later
 * needs a new stack; the memory must stay valid until moe_stack_destroy.
 * Shapes the stack kernel holds: H a multiple of 512 up to 2048, I a multiple
 * of 128 up to 4096 with I/32 in {12, 16, 32, 48, 64} (I = 384, 512, 1024,
 * 1536, 2048), top_k <= E <= 256 and E <= the SM count; sym8 layers and
 * stacks that mix formats are not taken.  Errors: ARG (including a shape or
 * format outside that set: run the
 * layers with moe_layer_ex instead), NOT_LOADED, NOT_DEVICE, ALIGN,
 * UNSUPPORTED, CUDA. */
MOE_API int moe_stack_create(const moe_handle_t *layers, int n_layers,
                             const uint16_t *const *router_w,
                             const float *const *router_bias, moe_stack_t *out);

/* Release the stack (host memory only; no device synchronisation).  Work
 * already enqueued keeps the pointers it was given.  NULL is a no-op. */
MOE_API int moe_stack_destroy(moe_stack_t s);

/* Bytes of device workspace the stack needs (tagged exchange words, one
 * 4-word piece or one router logit per 128-byte line, launch counters,
 * status; 140,544 bytes for H 2048, I 1536, E 64, top-4).  Errors: ARG. */
MOE_API int moe_stack_workspace_bytes(moe_stack_t s, size_t *bytes);

/* Give the stack its device workspace (caller-owned, 256-byte aligned, at
 * least moe_stack_workspace_bytes).  Zeroes it synchronously.  One
 * workspace serves one stack, and its decode calls must be ordered on the
 * GPU (one stream, or explicit dependencies): calls that overlap race on
 * the exchange words.  Errors: ARG, NOT_DEVICE, ALIGN, WORKSPACE, CUDA. */
MOE_API int moe_stack_set_workspace(moe_stack_t s, void *workspace, size_t bytes);

/* One decode step of one token.  r: device BF16 [H], the residual stream,
 * read as the first layer's input and overwritten with the last layer's
 * output.  Optional outputs (device, or NULL): r_hist BF16 [n_layers][H]
 * (each layer's input r), xn_hist BF16 [n_layers][H] (each layer's routed
 * vector), logits FP32 [n_layers][E], topk_ids int32 [n_layers][top_k],
 * topk_w FP32 [n_layers][top_k].  Enqueues one kernel on `stream`: no
 * allocation, no synchronisation, capturable in a CUDA graph.  Needs every
 * SM of the device free for the kernel (the launch fails with CUDA
 * otherwise).  Errors: ARG, NOT_LOADED (no workspace), NOT_DEVICE, ALIGN,
 * CUDA. */
MOE_API int moe_stack_decode(moe_stack_t s, uint16_t *r, uint16_t *r_hist,
                             uint16_t *xn_hist, float *logits,
                             int32_t *topk_ids, float *topk_w, void *stream);

/* Synchronise `stream`, return the stack's device status word
 * (MOE_DEVICE_* bits) in *device_status and clear it.  After
 * MOE_DEVICE_TIMEOUT the outputs of that step are invalid (r may hold the
 * step's input or a partial result); later steps run normally.
 * Errors: ARG, NOT_LOADED, CUDA. */
MOE_API int moe_stack_get_status(moe_stack_t s, void *stream, unsigned *device_status);

/* Test hook: the number of polls after which a wait on another CTA's tagged
 * words gives up (default 2^20; 0 makes every such wait give up at once).
 * Waits on the CTA's own copies in flight keep their full bound, so no copy
 * outlives a launch that gave up.  Errors: ARG. */
MOE_API int moe_stack_set_spin_limit(moe_stack_t s, int polls);

/* Profiling hook: when trace is a device buffer of at least
 * n_layers * SMs * 16 * 8 bytes (SMs = the device's multiprocessor count),
 * every later moe_stack_decode writes, per layer l and CTA b, sixteen
 * global-timer stamps (ns) at trace[(l * SMs + b) * 16 + slot]: 0 layer
 * start, 1 layer input gathered, 2 router logit published, 3 all logits
 * gathered, 10 top-k done, 4 down-row copies issued, 9 first gate/up rows
 * loaded (thread 0), 5 gate/up of the CTA done, 6 all of h gathered,
 * 15 h staged, 7 down GEMV done, 8 layer output published; slots 11..14
 * unused.  NULL turns it off.
 * Errors: ARG, WORKSPACE (buffer too small), NOT_DEVICE, ALIGN. */
MOE_API int moe_stack_set_trace(moe_stack_t s, unsigned long long *trace, size_t bytes);

/* ---------------------------------------------------------------------
 * Forward without any device allocation.  No counterpart in the paper: this
 * entry point exists for callers that may not call cudaMalloc -- code that
 * runs inside another framework's memory pool or allocator callback, or
 * hosts whose device memory is budgeted and accounted elsewhere.  It computes
 * exactly what moe_create + moe_load_packed + moe_set_workspace +
 * moe_forward_ex(residual) compute, with the same kernels, but without a
 * handle: its scratch (status word, SwiGLU activations h) lives in one
 * file-scope device array of MOE_NOALLOC_SCRATCH_BYTES bytes that every GPU
 * loading this library holds until the process exits.
 *
 * Limit (beyond it the call returns MOE_ERR_WORKSPACE and enqueues
 * nothing): T * top_k * I * 2 <= MOE_NOALLOC_MAX_H_BYTES.  Shapes as for
 * moe_create.
 * Arguments: codes_u8 / scales_e8m0 as for moe_load_packed (device,
 * contiguous [E][3][...], 16-byte aligned, read in place); x, topk_ids,
 * topk_w, residual (or NULL; may alias y), y as for moe_forward_ex.  These
 * pointers are not checked to be device memory (that check would itself be
 * a runtime call per pointer); they must be, and must hold the sizes the
 * shape implies.
 * The first call on a device (with that device current) looks up the
 * scratch's device address with cudaGetSymbolAddress (a runtime call, made
 * once per device).  Every call enqueues its kernels on `stream`
 * and shares the one scratch array: calls that overlap on the GPU
 * (different streams, or different threads without ordering) race on it.
 * The kernels report an id outside [0, E) (that slot contributes 0) or a
 * bounded wait that gave up in the scratch's status word; it accumulates
 * over calls until moe_forward_noalloc_status reads and clears it.
 * Errors: ARG, ALIGN, WORKSPACE, UNSUPPORTED, CUDA. */
#define MOE_NOALLOC_MAX_H_BYTES (512u * 1024u)
#define MOE_NOALLOC_SCRATCH_BYTES (256u + MOE_NOALLOC_MAX_H_BYTES)
MOE_API int moe_forward_noalloc(int E, int H, int I, int top_k,
                                const uint8_t *codes_u8,
                                const uint8_t *scales_e8m0, const uint16_t *x,
                                int T, const int32_t *topk_ids,
                                const float *topk_w, const uint16_t *residual,
                                uint16_t *y, void *stream);

/* Device status word of moe_forward_noalloc on the current device
 * (MOE_DEVICE_* bits, accumulated since the last read): synchronises
 * `stream`, copies the word to *device_status and clears it (no
 * allocation).  Errors: ARG, UNSUPPORTED, CUDA. */
MOE_API int moe_forward_noalloc_status(void *stream, unsigned *device_status);

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char *moe_status_string(int status);

/* MOE_OK if the current device is sm_100 (B200), else MOE_ERR_UNSUPPORTED
 * or MOE_ERR_CUDA. */
MOE_API int moe_device_check(void);

/* Test hook: dequantise n packed elements (n % 32 == 0) with the same
 * in-register decode the GEMV kernels use; out[j] = E2M1(code j) *
 * 2^(scales[j/32]-127) in FP32.  codes device uint8 [n/2], scales device
 * uint8 [n/32], out device FP32 [n].  Errors: ARG, NOT_DEVICE, ALIGN, CUDA.
 */
MOE_API int moe_debug_dequant(const uint8_t *codes, const uint8_t *scales, int64_t n,
                      float *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MXFP4_H */
