// sym8.cu — experts in the sym8 format on the per-(token, slot) GEMV path
// (up to 4 tokens; larger batches take the grouped mma.sync tiles of
// grouped.cu, unless asked for this path or the scales are not 4-byte
// aligned).
//
// Source: page "LFM2.5-8B-A1B — Core AI (.aimodel)", table "Provenance", row
// "Weight format": symmetric-linear int8 weights with one scale per K-block of
// 32.  Read here as: one two's-complement byte q per weight, one IEEE binary16
// scale s per 32 consecutive K elements of a row, w = q s, no zero point.
// Everything else is the packed-MXFP4 layer's arithmetic (model card
// "LFM2.5-24B-A2B — Packed MXFP4 Inference": "Grouped top-4 expert execution"
// for gate/up, SwiGLU, down and the sequential BF16 combine; table "Model and
// quantization" for BF16 activations, FP32 accumulation, BF16 outputs).
//
// Layout (as moe_load_packed_sym8 binds it): codes [E][3][rows][K] int8,
// scales [E][3][rows][K/32] little-endian binary16 words; matrix m of expert e
// is read through the handle's device table, in place.
//
// Arithmetic.  A weight byte becomes an FP32 value exactly by a byte permute
// into the float 2^23 + (q + 128) followed by one subtraction of 2^23 + 128;
// BF16 activations widen to FP32 exactly; each product q x is exact in FP32
// (8 x 8 significant bits).  A lane sums the 16 products of its 16-byte chunk
// in FP32, scales that half-group sum by the block's s (binary16 -> FP32
// exact) and adds it to its running sum; the warp then adds its lanes' sums.
// g and u are rounded to BF16, SiLU(g) to BF16, h = BF16(SiLU(g) u); the down
// sums give o = BF16(sum), and the combine is the sequential BF16 one
// (wb = BF16(w), y = BF16(y + BF16(o wb)), then y = BF16(r + y)).
//
// Two launches per chunk of up to kS8MaxT tokens, in the layer's programmatic
// launch chain: gate/up + SwiGLU (a warp takes kS8GuItems consecutive
// (pair, row) items per step and streams their gate and up rows together,
// the tokens' x staged in shared memory) writing h to the workspace, then
// down + combine + residual (one warp per (token, output row), the down rows
// of up to kS8DownSlots slots streamed together, the chunk's h staged in
// shared memory).  Lane l takes the 16-byte chunks l, l + 32, ... of a row:
// per row the sums and their order do not depend on how many rows stream
// together.  An expert id outside [0, E) gives that slot h = 0 and o = 0 and
// sets the status word's bad-id bit.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gemv.cuh"  // kernels.cuh, launch_ex

namespace moe {

namespace {

constexpr int kS8Threads = 256;
constexpr int kS8Warps = kS8Threads / 32;
constexpr int kS8CtasPerSm = 4;  // warps in flight per SM: 32 (streaming GEMV)
constexpr int kS8DownSlots = 4;  // slots whose down rows one warp streams together
#ifndef MOE_S8_GU_ITEMS
#define MOE_S8_GU_ITEMS 2
#endif
constexpr int kS8GuItems = MOE_S8_GU_ITEMS;  // gate/up items one warp streams together

// Four int8 weights of one 32-bit word (byte 0 = lowest K index) -> FP32,
// exactly: byte i, biased to q + 128, becomes the low byte of the float with
// bit pattern 0x4B0000xx = 2^23 + xx.
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float (&f)[4]) {
    const uint32_t u = w ^ 0x80808080u;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u | (unsigned)i)) - 8388736.0f;
}

// Sum of the 16 products of one 16-byte chunk of weights with 16 BF16
// activations (two 16-byte pieces, lower K first), in K order.
__device__ __forceinline__ float s8_chunk_dot(const uint4 &wq, const uint4 &x0, const uint4 &x1) {
    const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
    const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float f[4];
        s8x4_to_f32(wv[i], f);
        acc = fmaf(f[0], __uint_as_float(xv[2 * i] << 16), acc);
        acc = fmaf(f[1], __uint_as_float(xv[2 * i] & 0xFFFF0000u), acc);
        acc = fmaf(f[2], __uint_as_float(xv[2 * i + 1] << 16), acc);
        acc = fmaf(f[3], __uint_as_float(xv[2 * i + 1] & 0xFFFF0000u), acc);
    }
    return acc;
}

// The routing of the launch's tokens into shared memory: the given ids and
// weights, or (logits given) the softmax top-k of each token's logits by
// warp 0, the warp_topk that the standalone top-k kernel runs (same ids and
// weights); gate/up CTA 0 also writes them out when asked.  All threads; ends
// with a CTA barrier.
__device__ __forceinline__ void s8_routing(const Sym8Params &p, int *s_ids, float *s_w,
                                           bool write_out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k;
    if (p.logits) {
        if (warp == 0) {
            #pragma unroll 1
            for (int t = 0; t < p.T; ++t) {
                int id;
                float w;
                warp_topk_any(p.logits + (size_t)t * p.E, p.E, k, lane, id, w);
                if (lane < k) {
                    s_ids[t * k + lane] = id;
                    s_w[t * k + lane] = w;
                    if (write_out && p.ids_out) {
                        p.ids_out[t * k + lane] = id;
                        p.w_out[t * k + lane] = w;
                    }
                }
            }
        }
    } else {
        for (int i = tid; i < p.T * k; i += kS8Threads) {
            s_ids[i] = p.ids[i];
            s_w[i] = p.w[i];
        }
    }
    __syncthreads();
}

// binary16 block scale of the 16-byte chunk c of a row (two chunks per block).
__device__ __forceinline__ float s8_scale(const uint8_t *row_scales, int c) {
    const uint16_t *s = reinterpret_cast<const uint16_t *>(row_scales);
    return f16_bits_to_f32(__ldg(s + (c >> 1)));
}

// gate/up + SwiGLU.  Item (q, i): pair q = t k + j (token t, slot j), row i of
// the expert's gate and up matrices; h[q][i] = BF16(BF16(SiLU(BF16(g))) BF16(u)).
__global__ void __launch_bounds__(kS8Threads) sym8_gateup_kernel(const Sym8Params p) {
    extern __shared__ __align__(16) uint4 s_x[];  // [T][H/8]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_ids[kS8MaxT * kMaxTopK];
    __shared__ float s_w[kS8MaxT * kMaxTopK];
    pdl_wait();  // x and the routing come from earlier kernels
    pdl_launch_dependents();
    const int H = p.H, I = p.I, k = p.k, E = p.E;
    const int np8 = H >> 3;
    const uint4 *x = reinterpret_cast<const uint4 *>(p.x);
    for (int i = tid; i < p.T * np8; i += kS8Threads) s_x[i] = x[i];
    s8_routing(p, s_ids, s_w, blockIdx.x == 0);
    const size_t rs = (size_t)H >> 4;  // scale bytes of a row
    const long long items = (long long)p.T * k * I;
    // kS8GuItems consecutive items per warp per step: their gate and up rows
    // stream together (per row the same chunks, order and sums)
    #pragma unroll 1
    for (long long it0 = ((long long)blockIdx.x * kS8Warps + warp) * kS8GuItems; it0 < items;
         it0 += (long long)gridDim.x * kS8Warps * kS8GuItems) {
        const uint8_t *rg[kS8GuItems], *sg[kS8GuItems], *ru[kS8GuItems], *su[kS8GuItems];
        const uint4 *xs[kS8GuItems];
        bool ok[kS8GuItems];
#pragma unroll
        for (int d = 0; d < kS8GuItems; ++d) {
            const long long it = it0 + d;
            const int q = it < items ? (int)(it / I) : 0, i = it < items ? (int)(it - (long long)q * I) : 0;
            const int e = it < items ? s_ids[q] : -1;
            ok[d] = e >= 0 && e < E;
            if (it < items && !ok[d] && i == 0 && lane == 0) atomicOr(p.status, kBadExpertId);
            const ExpertPtrs *ep = ok[d] ? p.table + e : nullptr;
            rg[d] = ok[d] ? ep->codes[0] + (size_t)i * H : nullptr;
            sg[d] = ok[d] ? ep->scales[0] + (size_t)i * rs : nullptr;
            ru[d] = ok[d] ? ep->codes[1] + (size_t)i * H : nullptr;
            su[d] = ok[d] ? ep->scales[1] + (size_t)i * rs : nullptr;
            xs[d] = s_x + (size_t)(q / k) * np8;
        }
        float ag[kS8GuItems], au[kS8GuItems];
#pragma unroll
        for (int d = 0; d < kS8GuItems; ++d) ag[d] = au[d] = 0.f;
        const int nc = H >> 4;
        #pragma unroll 1
        for (int c = lane; c < nc; c += 32) {
            uint4 wg[kS8GuItems], wu[kS8GuItems];
#pragma unroll
            for (int d = 0; d < kS8GuItems; ++d)
                if (ok[d]) {
                    wg[d] = ld_stream16(rg[d] + (size_t)c * 16);
                    wu[d] = ld_stream16(ru[d] + (size_t)c * 16);
                }
#pragma unroll
            for (int d = 0; d < kS8GuItems; ++d)
                if (ok[d]) {
                    ag[d] = fmaf(s8_chunk_dot(wg[d], xs[d][2 * c], xs[d][2 * c + 1]), s8_scale(sg[d], c),
                                 ag[d]);
                    au[d] = fmaf(s8_chunk_dot(wu[d], xs[d][2 * c], xs[d][2 * c + 1]), s8_scale(su[d], c),
                                 au[d]);
                }
        }
#pragma unroll
        for (int d = 0; d < kS8GuItems; ++d) {
            const long long it = it0 + d;
            const float g0 = warp_sum(ag[d]), u0 = warp_sum(au[d]);
            if (lane == 0 && it < items) {
                uint16_t hv = 0;
                if (ok[d]) {
                    const float g = round_bf16(g0), u = round_bf16(u0);
                    const float sl = round_bf16(g / (1.0f + expf(-g)));
                    hv = f32_to_bf16(sl * u);
                }
                p.h[it] = hv;
            }
        }
    }
}

// down + combine + residual.  Item (t, n): output row n of token t; the
// slots' o_j = BF16(down row n . h_j) in slot order, combined sequentially in
// BF16, then the residual.  The slots' rows are streamed together (every
// slot's chunk c loaded before any of them is used); per row the chunks, their
// order and the sums are those of the one-row form (same bits).
__global__ void __launch_bounds__(kS8Threads) sym8_down_kernel(const Sym8Params p) {
    extern __shared__ __align__(16) uint4 s_h[];  // [T][k][I/8]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_ids[kS8MaxT * kMaxTopK];
    __shared__ float s_w[kS8MaxT * kMaxTopK];
    pdl_wait();  // h comes from the gate/up kernel
    pdl_launch_dependents();
    const int H = p.H, I = p.I, k = p.k, E = p.E;
    const int np8 = I >> 3;
    const uint4 *hg = reinterpret_cast<const uint4 *>(p.h);
    for (int i = tid; i < p.T * k * np8; i += kS8Threads) s_h[i] = hg[i];
    s8_routing(p, s_ids, s_w, false);
    const size_t rs = (size_t)I >> 4;
    const long long items = (long long)p.T * H;
    #pragma unroll 1
    for (long long it = (long long)blockIdx.x * kS8Warps + warp; it < items;
         it += (long long)gridDim.x * kS8Warps) {
        const int t = (int)(it / H), n = (int)(it - (long long)t * H);
        float y = 0.f;
        // slots in groups of kS8DownSlots, each group's rows streamed together
        #pragma unroll 1
        for (int j0 = 0; j0 < k; j0 += kS8DownSlots) {
            const uint8_t *rc[kS8DownSlots];
            const uint8_t *rsc[kS8DownSlots];
            bool ok[kS8DownSlots];
#pragma unroll
            for (int d = 0; d < kS8DownSlots; ++d) {
                const int j = j0 + d;
                const int e = j < k ? s_ids[t * k + j] : -1;
                ok[d] = e >= 0 && e < E;
                if (j < k && !ok[d] && lane == 0 && n == 0) atomicOr(p.status, kBadExpertId);
                rc[d] = ok[d] ? p.table[e].codes[2] + (size_t)n * I : nullptr;
                rsc[d] = ok[d] ? p.table[e].scales[2] + (size_t)n * rs : nullptr;
            }
            float acc[kS8DownSlots];
#pragma unroll
            for (int d = 0; d < kS8DownSlots; ++d) acc[d] = 0.f;
            const int nc = I >> 4;
            #pragma unroll 1
            for (int c = lane; c < nc; c += 32) {
                uint4 wq[kS8DownSlots];
#pragma unroll
                for (int d = 0; d < kS8DownSlots; ++d)
                    if (ok[d]) wq[d] = ld_stream16(rc[d] + (size_t)c * 16);
#pragma unroll
                for (int d = 0; d < kS8DownSlots; ++d)
                    if (ok[d]) {
                        const uint4 *hs = s_h + (size_t)(t * k + j0 + d) * np8;
                        acc[d] = fmaf(s8_chunk_dot(wq[d], hs[2 * c], hs[2 * c + 1]),
                                      s8_scale(rsc[d], c), acc[d]);
                    }
            }
#pragma unroll
            for (int d = 0; d < kS8DownSlots; ++d) {
                const int j = j0 + d;
                if (j >= k) break;
                const int q = t * k + j;
                const float a = warp_sum(acc[d]);
                const float o = ok[d] ? round_bf16(a) : 0.f;
                if (lane == 0 && p.o_keep) p.o_keep[(size_t)q * H + n] = f32_to_bf16(o);
                const float wb = round_bf16(s_w[q]);
                y = round_bf16(y + round_bf16(o * wb));
            }
        }
        if (lane == 0) {
            if (p.residual) y = round_bf16(bf16_to_f32(p.residual[it]) + y);
            p.y[it] = f32_to_bf16(y);
        }
    }
}

size_t s8_gateup_smem(int T, int H) { return (size_t)T * H * 2; }
size_t s8_down_smem(int T, int k, int I) { return (size_t)T * k * I * 2; }

PerDeviceOnce g_s8_attr;

}  // namespace

bool sym8_supported(int H, int I, int k) {
    return H >= 32 && I >= 32 && H % 32 == 0 && I % 32 == 0 && k >= 1 && k <= kMaxTopK &&
           s8_gateup_smem(1, H) <= kS8SmemMax && s8_down_smem(1, k, I) <= kS8SmemMax;
}

int sym8_max_chunk(int H, int I, int k) {
    int c = kS8MaxT;
    while (c > 1 && (s8_gateup_smem(c, H) > kS8SmemMax || s8_down_smem(c, k, I) > kS8SmemMax)) --c;
    return c;
}

cudaError_t launch_sym8(const Sym8Params &p, int num_sms, bool run_gu, bool run_dn,
                        cudaStream_t s, bool pdl) {
    if (p.T < 1 || p.T > kS8MaxT || !sym8_supported(p.H, p.I, p.k)) return cudaErrorInvalidValue;
    const size_t sg = s8_gateup_smem(p.T, p.H), sd = s8_down_smem(p.T, p.k, p.I);
    if (sg > kS8SmemMax || sd > kS8SmemMax) return cudaErrorInvalidValue;
    cudaError_t e = per_device_once(g_s8_attr, [] {
        cudaError_t r = cudaFuncSetAttribute(sym8_gateup_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kS8SmemMax);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(sym8_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kS8SmemMax);
    });
    if (e != cudaSuccess) return e;
    const int grid = num_sms * kS8CtasPerSm;
    if (run_gu && (e = launch_ex(sym8_gateup_kernel, dim3(grid), dim3(kS8Threads), sg, s, pdl, p)) !=
                      cudaSuccess)
        return e;
    if (run_dn && (e = launch_ex(sym8_down_kernel, dim3(grid), dim3(kS8Threads), sd, s, pdl, p)) !=
                      cudaSuccess)
        return e;
    return cudaSuccess;
}

}  // namespace moe
