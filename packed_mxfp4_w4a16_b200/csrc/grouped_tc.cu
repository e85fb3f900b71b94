// grouped_tc.cu — the grouped expert products on the 5th-generation tensor
// cores (tcgen05.mma with TMEM accumulators), for batches whose experts see
// many tokens each (large prefill chunks).
//
// Sources: model card "LFM2.5-24B-A2B — Packed MXFP4 Inference", "Grouped
// top-4 expert execution" (grouped gate / up / down products, activation and
// multiplication) and table "Model and quantization" (E2M1 + E8M0 per 32,
// BF16 activations, FP32 accumulation); page "LFM2.5-8B-A1B — Core AI
// (.aimodel)", section "Provenance" (the batched path sorts the (token,
// expert) pairs so that each expert's tokens form one group).
//
// One CTA per (128 rows of a matrix, expert), 16 conversion warps and one
// MMA / TMA warp.  The CTA walks K in tiles of 64.  The packed codes of each
// tile (128 rows x 32 bytes per matrix) arrive by one TMA tensor load into a
// ring of shared-memory slots, several tiles ahead (mbarrier completion); per
// tile, the threads (four per row, a quarter of the tile's K each) dequantise
// the 128 x 64 packed weights of each matrix into BF16 (code x 2^(e-127),
// exact in BF16: the E8M0 scale is folded into A, so the tensor core
// accumulates the whole K range in FP32 without a per-group step; NVFP4
// weights, page "primitive-ai/LFM2.5-24B-A2B-NVFP4A16": code x its 16-element
// block's E4M3 scale, also exact, the expert's FP32 multiplier applied to the
// accumulator in the epilogue) and copy
// the BF16 activation rows of up to 128 tokens of the expert (B, in a ring of
// its own, two tiles ahead), both into shared memory in the
// K-major core-matrix layout (8 rows x 16 bytes per core matrix).  One thread
// then issues the tile's 4 x NMAT tcgen05.mma (M = 128, N = tokens rounded up
// to 16, at most 128, K = 16, BF16 x BF16 -> FP32 in TMEM) and commits them to the tile's
// mbarrier; two tiles alternate, so the dequantisation of one overlaps the
// products of the other.  The epilogue reads the accumulators from TMEM
// (tcgen05.ld: warp w reads rows 32 (w % 4) .. + 31, the (w / 4)-th quarter
// of the token columns) and applies the same
// rounding points as the other paths: h = BF16(BF16(silu(BF16(g))) BF16(u))
// for gate / up, o = BF16(acc) for down.  Products are exact in FP32; only
// the FP32 summation order differs from the oracle.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "gemv.cuh"

namespace moe {

namespace {

constexpr int kTcM = 128;          // matrix rows per CTA (MMA M)
constexpr int kTcK = 64;           // K per shared-memory tile (4 MMAs of K = 16)
constexpr int kTcMaxN = 128;       // tokens per pass (MMA N <= 128, a multiple of 16)
constexpr int kTcWork = 512;       // conversion threads: 4 per weight row, 16 warps
constexpr int kTcThreads = kTcWork + 32;  // + the MMA / TMA warp
constexpr uint32_t kTcTileA = kTcM * kTcK * 2;    // 16 KB of BF16 per matrix
constexpr uint32_t kTcTileB = kTcMaxN * kTcK * 2; // 16 KB of BF16
constexpr int kTcBSlots = 4;                      // B tiles in flight (ring)
constexpr size_t kTcSmemBudget = 220 * 1024;      // dynamic shared memory of a CTA

__host__ __device__ constexpr uint32_t tc_stage_bytes(int nmat) {
    return (uint32_t)nmat * kTcTileA;  // an MMA stage holds the A tiles
}

// Byte offset of element (row, k) of a K-major tile with 64 K per row: core
// matrices of 8 rows x 8 elements (16 bytes per row, 128 bytes each); the 8
// K-chunks of a group of 8 rows lie 128 bytes apart (leading byte offset),
// groups of 8 rows 1024 bytes apart (stride byte offset).
__device__ __forceinline__ uint32_t tc_off(int row, int kchunk) {
    return (uint32_t)(row >> 3) * 1024u + (uint32_t)kchunk * 128u + (uint32_t)(row & 7) * 16u;
}

// Shared-memory matrix descriptor: no swizzle, K-major; start address,
// leading byte offset 128 (next K-chunk), stride byte offset 1024 (next 8
// rows), all in 16-byte units; version 1 (bits 46..47).
__device__ __forceinline__ uint64_t tc_desc(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
           ((uint64_t)(1024u >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: FP32 accumulator (bits 4..5 = 1),
// A and B BF16 (bits 7..9 and 10..12 = 1), both K-major, N / 8 at bit 17,
// M / 16 at bit 24.
__device__ __forceinline__ uint32_t tc_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kTcM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrive on *bar once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy shared-memory writes -> visible to the tensor core.
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 lanes x 32 bits x 8 columns of TMEM: lane l of the warp gets row
// (taddr lane field + l), columns taddr .. taddr + 7.
__device__ __forceinline__ void tc_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp_async16_tc(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 8 E2M1 codes (one 4-byte word) times the scale sf -> 8 BF16 (exact: the
// products have at most 2 significant bits).
__device__ __forceinline__ uint4 dequant8_bf16(uint32_t w, float sf) {
    uint32_t h[4];
    e2m1x8_to_f16x8(w, h);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = pack_bf16x2(f16_bits_to_f32(h[i] & 0xFFFFu) * sf, f16_bits_to_f32(h[i] >> 16) * sf);
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Barrier of the conversion threads alone (named barrier 1; every
// conversion warp executes it, the MMA warp does not).
__device__ __forceinline__ void conv_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kTcWork) : "memory");
}

__device__ __forceinline__ const uint8_t *tc_scales(const GroupedParams &p, int e, int m) {
    return p.codes_base ? p.scales_base + (size_t)(3 * e + m) * p.scales_stride
                        : p.table[e].scales[m];
}

}  // namespace

namespace {

constexpr int kTcRaw = 4;  // packed K tiles in flight (TMA ring slots)
constexpr uint32_t kTcRawSlot = kTcM * 32;  // bytes of one matrix's packed tile

// Shared-memory plan of one CTA (dynamic part): 2 MMA stages of A tiles
// (NMAT x 16 KB BF16); the B ring [kTcBSlots][16 KB BF16]; the packed codes
// ring [kTcRaw][NMAT][128 rows][32 bytes]; the CTA's scale rows
// [NMAT][128][K/32].
__host__ __device__ constexpr uint32_t tc_b_off(int nmat) { return 2 * tc_stage_bytes(nmat); }
__host__ __device__ constexpr uint32_t tc_raw_off(int nmat) {
    return tc_b_off(nmat) + (uint32_t)kTcBSlots * kTcTileB;
}
__host__ __device__ constexpr uint32_t tc_sc_off(int nmat) {
    return tc_raw_off(nmat) + (uint32_t)kTcRaw * nmat * kTcRawSlot;
}
// Scale rows: K/32 E8M0 bytes, or K/16 E4M3 bytes (nv).  Then, when the plan
// has room for it ([pairs] ints: a group holds at most all the launch's T k
// pairs), the B row of every token of the group; else the kernel reads the
// rows from the sorted pair list in global memory.
__host__ __device__ inline uint32_t tc_src_off(int nmat, int K, int nv) {
    return tc_sc_off(nmat) + (uint32_t)nmat * kTcM * (uint32_t)(K / (nv ? 16 : 32));
}
__host__ __device__ inline uint32_t tc_smem_bytes(int nmat, int K, int pairs, int nv) {
    return tc_src_off(nmat, K, nv) + (uint32_t)pairs * sizeof(int);
}

// One TMA tile load of the 3-D code tensor (x: byte in the row, y: row,
// z: matrix 3 e + m) into shared memory, completing on *bar.  Loads only
// this GPU's memory, into this CTA alone.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// Bounded wait on phase `parity` of *bar that also gives up once *abort is
// set; a timeout sets *abort, so every other wait of the CTA ends too.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, unsigned parity, volatile int *abort) {
    #pragma unroll 1
    for (int i = 0; i < kMaxSpin; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
    }
    *abort = 1;
    return false;
}

// Warp-specialised: warps 0..15 convert (A tiles, B copies, epilogue), warp
// 16 (lane 0) issues the TMA loads of the packed codes and the MMAs.  Stage
// hand-offs: s_full[s] (16 conversion-warp arrivals: A and B of the tile are
// in shared memory), s_mma[s] (tcgen05.commit: the tile's products are done,
// the stage may be rewritten), s_raw[j] (TMA bytes of ring slot j), s_tfree
// (16 arrivals: the pass's accumulators were read).
// NV: NVFP4 weights: A = code x its 16-element block's E4M3 scale (exact in
// BF16: at most 6 significant bits), the expert's FP32 multiplier applied to
// the accumulator in the epilogue (one FP32 rounding before the BF16 one).
// TAB: the token-row table in shared memory (else read from the sorted pair
// list in global memory).
template <int NMAT, bool NV, bool TAB>
__global__ void __launch_bounds__(kTcThreads, 1)
grouped_tc_kernel(const GroupedParams p, const __grid_constant__ CUtensorMap codes_map) {
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t s_full[2];
    __shared__ __align__(8) uint64_t s_mma[2];
    __shared__ __align__(8) uint64_t s_raw[kTcRaw];
    __shared__ __align__(8) uint64_t s_tfree;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int e = blockIdx.y;
    pdl_wait();
    pdl_launch_dependents();
    const int seg0 = p.offs[e], n_e = p.offs[e + 1] - seg0;
    if (n_e <= 0) return;  // uniform: no token chose this expert (no TMEM taken)

    const int K = NMAT == 2 ? p.H : p.I;  // reduction length
    const int M = NMAT == 2 ? p.I : p.H;  // matrix rows (a multiple of 128)
    const int row0 = blockIdx.x * kTcM;
    const int nkt = K / kTcK;
    const int npass = (n_e + kTcMaxN - 1) / kTcMaxN;
    const int total = npass * nkt;  // (pass, K tile) iterations
    const uint32_t rs = (uint32_t)K >> (NV ? 4 : 5);  // scale bytes per row
    uint8_t *raw = sm + tc_raw_off(NMAT);
    uint8_t *scl = sm + tc_sc_off(NMAT);
    // per token of the group: its B row (x row of the pair's token, or h row
    // of the pair), in shared memory when the launch's plan holds the table
    int *s_src = reinterpret_cast<int *>(sm + tc_src_off(NMAT, K, NV ? 1 : 0));

    if (warp == 0) {  // TMEM: NMAT x 128 FP32 columns x 128 lanes
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&s_tmem)), "r"(NMAT * kTcMaxN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&s_full[0], kTcWork / 32);
        mbar_init(&s_full[1], kTcWork / 32);
        mbar_init(&s_mma[0], 1);
        mbar_init(&s_mma[1], 1);
#pragma unroll
        for (int j = 0; j < kTcRaw; ++j) mbar_init(&s_raw[j], 1);
        mbar_init(&s_tfree, kTcWork / 32);
        s_abort = 0;
        mbar_fence_init();
    }
    for (int i = tid; TAB && i < n_e; i += kTcThreads) {
        const int pr = p.perm[seg0 + i];
        s_src[i] = NMAT == 2 ? pr / p.k : pr;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort = &s_abort;

    if (warp == kTcWork / 32) {
        // ---- MMA + TMA warp: lane 0 issues, the other lanes wait at the end ----
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&codes_map))
                         : "memory");
            const uint64_t pol = l2_evict_first_policy();  // packed rows are read once
            int raw_next = 0;
            auto issue_raw = [&](int it) {
                raw_next = it + 1;
                const int j = it % kTcRaw, kt = it % nkt;
                mbar_arrive_expect_tx(&s_raw[j], (unsigned)(NMAT * kTcRawSlot));
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
                    tma_load_3d(raw + ((uint32_t)j * NMAT + m) * kTcRawSlot, &codes_map, kt * 32,
                                row0, 3 * e + (NMAT == 2 ? m : 2), &s_raw[j], pol);
            };
            for (int j = 0; j < kTcRaw && j < total; ++j) issue_raw(j);
            int issued = 0;
            #pragma unroll 1
            for (int it = 0; it < total; ++it) {
                const int s = it & 1, pass = it / nkt, kt = it % nkt;
                const int nt = min(kTcMaxN, n_e - pass * kTcMaxN);
                if (!tc_wait(&s_full[s], (unsigned)(it >> 1) & 1u, abort)) break;
                // the first tile of a pass overwrites the accumulators: the
                // previous pass's epilogue must have read them
                if (kt == 0 && pass > 0 && !tc_wait(&s_tfree, (unsigned)(pass - 1) & 1u, abort))
                    break;
                tc_fence_after();
                const uint32_t idesc = tc_idesc((nt + 15) & ~15);
                const uint32_t b_addr =
                    smem_u32(sm + tc_b_off(NMAT) + (uint32_t)(it % kTcBSlots) * kTcTileB);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint32_t a_addr =
                        smem_u32(sm + (uint32_t)s * tc_stage_bytes(NMAT) + (uint32_t)m * kTcTileA);
#pragma unroll
                    for (int kk = 0; kk < kTcK / 16; ++kk)
                        tc_mma(tmem + (uint32_t)(m * kTcMaxN), tc_desc(a_addr + kk * 256),
                               tc_desc(b_addr + kk * 256), idesc, kt > 0 || kk > 0);
                }
                tc_commit(&s_mma[s]);
                issued = it + 1;
                // ring slot it % kTcRaw was read by every conversion thread
                // before its s_full arrival: refill it
                if (it + kTcRaw < total) issue_raw(it + kTcRaw);
            }
            // nothing in flight at exit (bounded): the products issued, the
            // last packed loads (one per ring slot; earlier ones were consumed)
            if (issued > 0) mbar_wait(&s_mma[(issued - 1) & 1], (unsigned)((issued - 1) >> 1) & 1u);
            for (int j = max(0, raw_next - kTcRaw); j < raw_next; ++j)
                mbar_wait(&s_raw[j % kTcRaw], (unsigned)(j / kTcRaw) & 1u);
        }
        __syncwarp();
    } else {
        // ---- conversion warps ----
        // this thread's row and K quarter (a warp covers 8 consecutive rows:
        // its reads of the packed ring are contiguous)
        const int rrow = tid >> 2, quarter = tid & 3;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const int mat = NMAT == 2 ? m : 2;
            const uint8_t *gsc = tc_scales(p, e, mat) + (size_t)(row0 + rrow) * rs;
            // K / 32 and K / 16 are multiples of 4 (K % 128 == 0): the row's
            // scales in 4-byte pieces, spread over its four threads
            for (uint32_t c = 4 * quarter; c < rs; c += 16)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                                 smem_u32(scl + ((uint32_t)m * kTcM + rrow) * rs + c)),
                             "l"(gsc + c)
                             : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // B rows of iteration it (its pass's tokens, K tile kt) into ring
        // slot it % kTcBSlots
        const uint16_t *bbase = NMAT == 2 ? p.x : p.h;
        auto issue_b = [&](int it) {
            const int pass = it / nkt, kt = it % nkt;
            const int tc = pass * kTcMaxN, nt = min(kTcMaxN, n_e - tc);
            uint8_t *b = sm + tc_b_off(NMAT) + (uint32_t)(it % kTcBSlots) * kTcTileB;
            // 64 consecutive i cover 8 rows x 8 chunks, row fastest: the 8
            // lanes of each shared-memory phase write 8 different rows of a
            // core matrix (distinct banks); each row gets 64 contiguous bytes
            // per warp from global memory
            for (int i = tid; i < ((nt + 7) & ~7) * 8; i += kTcWork) {
                const int n = ((i >> 6) << 3) | (i & 7), c = (i >> 3) & 7;
                if (n < nt) {
                    int src;
                    if (TAB) {
                        src = s_src[tc + n];
                    } else {
                        const int pr = p.perm[seg0 + tc + n];
                        src = NMAT == 2 ? pr / p.k : pr;
                    }
                    cp_async16_tc(b + tc_off(n, c), bbase + (size_t)src * K + kt * kTcK + c * 8);
                }
            }
        };
        // copy groups: {scales}, {B(0)}, {B(1)}, then one per iteration
        issue_b(0);
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (total > 1) issue_b(1);
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 2;" ::: "memory");
        // every row's scale bytes (copied by its four threads) visible to all
        conv_sync();
        #pragma unroll 1
        for (int it = 0; it < total; ++it) {
            const int s = it & 1, pass = it / nkt, kt = it % nkt;
            const int tc = pass * kTcMaxN, nt = min(kTcMaxN, n_e - tc);
            // A stage s and B slot (it + 2) % kTcBSlots were last read by the
            // products of iteration it - 2
            bool ok = it < 2 || tc_wait(&s_mma[s], (unsigned)((it - 2) >> 1) & 1u, abort);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (it + 2 < total) issue_b(it + 2);
            // all but the 2 newest groups: B of this iteration
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 2;" ::: "memory");
            ok = tc_wait(&s_raw[it % kTcRaw], (unsigned)(it / kTcRaw) & 1u, abort);
            if (!__all_sync(0xffffffffu, ok)) break;
            // ---- dequantise this thread's part of tile kt into stage s ----
            uint8_t *st = sm + (uint32_t)s * tc_stage_bytes(NMAT);
            const uint8_t *slot = raw + (uint32_t)(it % kTcRaw) * NMAT * kTcRawSlot;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                // K-chunks 2 q, 2 q + 1 of the row (8 code bytes: one E8M0
                // group, or exactly one 16-element E4M3 block)
                const uint2 cw = *reinterpret_cast<const uint2 *>(
                    slot + (uint32_t)m * kTcRawSlot + (uint32_t)rrow * 32 + 8 * quarter);
                const uint8_t *srow = scl + ((uint32_t)m * kTcM + rrow) * rs;
                float sf;
                if (NV) {
                    float hi_unused;
                    e4m3x2_to_f32(srow[4 * kt + quarter], sf, hi_unused);
                } else {
                    sf = e8m0_to_f32(srow[2 * kt + (quarter >> 1)]);
                }
                uint8_t *a = st + (uint32_t)m * kTcTileA;
                *reinterpret_cast<uint4 *>(a + tc_off(rrow, 2 * quarter)) = dequant8_bf16(cw.x, sf);
                *reinterpret_cast<uint4 *>(a + tc_off(rrow, 2 * quarter + 1)) = dequant8_bf16(cw.y, sf);
            }
            fence_async_shared();  // this thread's A and B writes -> the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_full[s]);
            if (kt == nkt - 1) {
                // ---- epilogue of this pass: accumulators -> outputs ----
                ok = tc_wait(&s_mma[s], (unsigned)(it >> 1) & 1u, abort);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const int lq = warp & 3;           // TMEM lane quarter of this warp
                const int r = row0 + lq * 32 + lane;  // this thread's matrix row
                const uint32_t lane_base = tmem + ((uint32_t)(lq * 32) << 16);
                const int N = (nt + 15) & ~15;
                // NVFP4: the expert's multiplier (gate/up or down)
                const float gm = NV ? __ldg(p.gscale + 2 * e + (NMAT == 2 ? 0 : 1)) : 1.0f;
                #pragma unroll 1
                for (int c0 = 8 * (warp >> 2); c0 < N; c0 += 32) {
                    float g[8], u[8];
                    tc_ld8(lane_base + (uint32_t)c0, g);
                    if (NMAT == 2) tc_ld8(lane_base + (uint32_t)(kTcMaxN + c0), u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int idx = tc + c0 + j;
                        if (idx >= tc + nt) continue;
                        const int pr = p.perm[seg0 + idx];
                        if (NMAT == 2) {
                            const float gv = round_bf16(NV ? g[j] * gm : g[j]);
                            const float uv = round_bf16(NV ? u[j] * gm : u[j]);
                            const float sl = round_bf16(gv / (1.0f + expf(-gv)));
                            p.h[(size_t)pr * M + r] = f32_to_bf16(sl * uv);
                        } else {
                            p.o[(size_t)pr * M + r] = f32_to_bf16(NV ? g[j] * gm : g[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_tfree);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // no copy in flight at exit
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && s_abort) atomicOr(p.status, kTimeoutStatus);
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(NMAT * kTcMaxN)
                     : "memory");
    }
}

}  // namespace

// ------------------------------------------------------------------ host --

namespace {

// The 3-D tensor map of the packed codes of one matrix kind: x = byte in a
// row (K / 2), y = row (M), z = matrix index 3 e + m over every expert;
// boxes of 32 bytes x 128 rows x 1 matrix.  Encoded once per (base, shape).
struct CodesMap {
    const void *base = nullptr;
    int E = 0, rows = 0, K = 0;
    CUtensorMap map;
};

PFN_cuTensorMapEncodeTiled encode_fn() {
    // looked up once (thread-safe static initialisation)
    static const PFN_cuTensorMapEncodeTiled fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
        return PFN_cuTensorMapEncodeTiled(nullptr);
    }();
    return fn;
}

cudaError_t codes_map(CodesMap &c, const uint8_t *base, size_t matrix_stride, int E, int rows,
                      int K) {
    if (c.base == base && c.E == E && c.rows == rows && c.K == K) return cudaSuccess;
    PFN_cuTensorMapEncodeTiled fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)K / 2, (cuuint64_t)rows, (cuuint64_t)3 * E};
    const cuuint64_t strides[2] = {(cuuint64_t)K / 2, (cuuint64_t)matrix_stride};
    const cuuint32_t box[3] = {32, (cuuint32_t)kTcM, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&c.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    c.base = base;
    c.E = E;
    c.rows = rows;
    c.K = K;
    return cudaSuccess;
}

// The map of the weights bound last, re-encoded when they change; the lock
// makes check, encode and copy one step for callers on several host threads
// (a launch never sees a map another thread is rewriting).
cudaError_t codes_map_copy(CodesMap &c, std::mutex &mu, const GroupedParams &p, int rows, int K,
                           CUtensorMap *out) {
    std::lock_guard<std::mutex> lock(mu);
    cudaError_t e = codes_map(c, p.codes_base, p.codes_stride, p.E, rows, K);
    if (e == cudaSuccess) *out = c.map;
    return e;
}

template <int NMAT, bool NV, bool TAB>
cudaError_t launch_tc_v(const GroupedParams &p, const CUtensorMap &map, size_t smem,
                        cudaStream_t s, bool pdl) {
    // the budget, once per device (the attribute belongs to the current
    // device's context)
    static PerDeviceOnce once;
    const cudaError_t attr = per_device_once(once, [] {
        return cudaFuncSetAttribute(grouped_tc_kernel<NMAT, NV, TAB>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kTcSmemBudget);
    });
    if (attr != cudaSuccess) return attr;
    const int M = NMAT == 2 ? p.I : p.H;
    return launch_ex(grouped_tc_kernel<NMAT, NV, TAB>, dim3(M / kTcM, p.E), dim3(kTcThreads), smem,
                     s, pdl, p, map);
}

template <int NMAT, bool NV>
cudaError_t launch_tc(const GroupedParams &p, const CUtensorMap &map, cudaStream_t s, bool pdl) {
    const int K = NMAT == 2 ? p.H : p.I;
    // the token-row table in shared memory when it fits beside the tiles
    const size_t with_table = tc_smem_bytes(NMAT, K, p.T * p.k, NV ? 1 : 0);
    if (with_table <= kTcSmemBudget)
        return launch_tc_v<NMAT, NV, true>(p, map, with_table, s, pdl);
    const size_t smem = tc_smem_bytes(NMAT, K, 0, NV ? 1 : 0);
    if (smem > kTcSmemBudget) return cudaErrorInvalidValue;
    return launch_tc_v<NMAT, NV, false>(p, map, smem, s, pdl);
}

}  // namespace

// The tensor-core products need the contiguous weight layout (one tensor map
// per matrix kind), H and I multiples of 128 and the shared-memory plan of
// both products within the budget.
bool grouped_tc_supported(int H, int I, int nv) {
    return H % 128 == 0 && I % 128 == 0 && tc_smem_bytes(2, H, 0, nv) <= kTcSmemBudget &&
           tc_smem_bytes(1, I, 0, nv) <= kTcSmemBudget;
}

namespace {

static_assert(sizeof(CUtensorMap) == sizeof(TcMapCache::map[0]), "opaque tensor-map bytes");

// The map of matrix kind `kind` from the handle's cache (encoded when the
// bound weights differ from the cached ones), else from the process-wide
// cache of the weights bound last.
cudaError_t kind_map(const GroupedParams &p, int kind, int rows, int K, CodesMap &shared,
                     std::mutex &mu, CUtensorMap *out) {
    if (!p.tc_maps) return codes_map_copy(shared, mu, p, rows, K, out);
    TcMapCache &c = *p.tc_maps;
    CUtensorMap *m = reinterpret_cast<CUtensorMap *>(c.map[kind]);
    if (c.base[kind] != p.codes_base || c.E[kind] != p.E || c.rows[kind] != rows ||
        c.K[kind] != K) {
        CodesMap fresh;
        const cudaError_t e = codes_map(fresh, p.codes_base, p.codes_stride, p.E, rows, K);
        if (e != cudaSuccess) return e;
        *m = fresh.map;
        c.base[kind] = p.codes_base;
        c.E[kind] = p.E;
        c.rows[kind] = rows;
        c.K[kind] = K;
    }
    *out = *m;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_grouped_tc_gateup(const GroupedParams &p, cudaStream_t s, bool pdl) {
    static CodesMap gu;
    static std::mutex mu;
    if (!p.codes_base) return cudaErrorInvalidValue;
    CUtensorMap map;
    cudaError_t e = kind_map(p, 0, p.I, p.H, gu, mu, &map);
    if (e != cudaSuccess) return e;
    return p.nv ? launch_tc<2, true>(p, map, s, pdl) : launch_tc<2, false>(p, map, s, pdl);
}

cudaError_t launch_grouped_tc_down(const GroupedParams &p, cudaStream_t s, bool pdl) {
    static CodesMap dn;
    static std::mutex mu;
    if (!p.codes_base) return cudaErrorInvalidValue;
    CUtensorMap map;
    cudaError_t e = kind_map(p, 1, p.H, p.I, dn, mu, &map);
    if (e != cudaSuccess) return e;
    return p.nv ? launch_tc<1, true>(p, map, s, pdl) : launch_tc<1, false>(p, map, s, pdl);
}

}  // namespace moe
