// The memory chain of both update rules, split into a parallel part and a short serial
// part (sm_100a).
//
// AI Wiki "Infini-Attention", "How does the compressive memory work?":
//   linear: M_s = M_{s-1} + sigma(K_s)^T V_s
//   delta : M_s = M_{s-1} + sigma(K_s)^T (V_s - sigma(K_s) M_{s-1} / den),
//           den_t = sigma(k_t) . z_{s-1}   (a row whose den is 0 predicts 0)
//   both  : z_s = z_{s-1} + sum_t sigma(k_t)
// The delta update is linear in M_{s-1}, and den needs only z_{s-1}, which never depends
// on M:
//   M_s = M_{s-1} + B_s - A_s M_{s-1},
//   B_s = sigma(K_s)^T V_s,   A_s = sigma(K_s)^T diag(1/den) sigma(K_s)   (d x d each).
// So the contractions over a segment's N tokens leave the serial path:
//   k_zsum      delta: per (chain, segment) dz_s = sum_t sigma(k_t), fp32 on the CUDA cores
//   k_zscan     per chain: z_{s-1} for every segment (what the segment kernel and den read)
//   k_mem_incr  per (chain, segment), all at once, on the tensor cores: B_s and (delta) A_s;
//               for the additive rule, whose increments do not need z, also dz_s as
//               sigma(K_s)^T 1 (the same two sigma parts against a tile of ones), so k is
//               read once on that path and k_zscan follows it
//   k_mem_chain delta: per (chain, 16 value columns), the recurrence in segment order, one
//               d x d x 32 product per segment on the tensor cores
//   k_mem_prefix linear: the running sum M0 + sum_{j<s} B_j, elementwise
// The last two write the bf16 snapshots M_{s-1} the segment kernel reads, and M_out.
//
// Precision: sigma(K) enters the contractions as two bf16 parts, sigma_hi = bf16(sigma) and
// sigma_lo = bf16(sigma - sigma_hi); with sigma ~ 1 a single bf16 rounding (2^-9) would
// cost about 5e-3 of M over 32 segments of 2048 tokens, the split about 3e-6.  The products
// are sigma_hi [V | W_hi] + sigma_lo [V | W_hi] + sigma_hi W_lo with W = diag(1/den) sigma
// split the same way (sigma_lo W_lo is below the fp32 rounding of the sums).  In the chain
// A_s and M_{s-1} are split too (three products).  z is summed in fp32: from sigma itself
// (delta), or from its two bf16 parts in an fp32 accumulator (additive).
// Rows of a short last segment past L carry sigma = 0 (not sigma(0) = 1): they add nothing.
// All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

// ---------------------------------------------------------------- z: column sums and prefix

// dz[chain * S + s][f] = sum over the rows t < L of segment s of sigma(k_t[f]).  One CTA per
// (chain, segment); thread (row lane, 8-feature chunk) reads 16-byte pieces of rows.
template <int D>
__global__ void __launch_bounds__(256)
k_zsum(const __nv_bfloat16 *__restrict__ k, float *__restrict__ dz, int64_t L, int N, int S)
{
    constexpr int CHK = D / 8;              // 16-byte chunks per row
    constexpr int RL = 256 / CHK;           // rows read side by side
    __shared__ float part[RL][D];
    const int64_t cs = blockIdx.x;
    const int64_t chain = cs / S;
    const int s = (int)(cs % S);
    const int ch = threadIdx.x % CHK, rl = threadIdx.x / CHK;
    const int64_t row0 = (int64_t)s * N;
    const int rows = (int)(L - row0 < N ? L - row0 : N);
    const uint4 *src = reinterpret_cast<const uint4 *>(k + (chain * L + row0) * D) + ch;
    // sigma = max(x + 1, e^min(x, 0)) (as elu1) with the multiply, the add and the sums on
    // packed fp32 pairs: the pass is bound by its instruction issue, not by HBM
    const uint64_t one2 = f2_pack(1.f, 1.f);
    const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
    uint64_t acc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = f2_pack(0.f, 0.f);
    // U rows per thread in flight: with few segments (one CTA each) the grid is small and
    // the loads in flight per thread set the bandwidth
    constexpr int U = 8;
    for (int r0 = rl; r0 < rows; r0 += U * RL) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (r0 + u * RL < rows) v[u] = __ldg(src + (int64_t)(r0 + u * RL) * CHK);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (r0 + u * RL >= rows) break;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
                float a0, a1, p0, p1;
                f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
                f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
                acc[e] = f2_add(acc[e], f2_pack(fmaxf(p0, ex2(a0)), fmaxf(p1, ex2(a1))));
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) f2_unpack(acc[e], part[rl][ch * 8 + 2 * e], part[rl][ch * 8 + 2 * e + 1]);
    __syncthreads();
    for (int f = threadIdx.x; f < D; f += 256) {
        float t = 0.f;
        for (int j = 0; j < RL; ++j) t += part[j][f];
        dz[cs * D + f] = t;
    }
}

// snapZ[chain * S + s] = z_{s-1} = z0 + sum_{j<s} dz_j for every segment, z_out = z_S.
// One CTA of 8 x D threads per chain: 8 groups of consecutive segments are summed side by
// side, then each group walks its segments again from the prefix of the groups before it.
// z0 is read before the first barrier, so z_out may alias it.
template <int D>
__global__ void __launch_bounds__(D * 8)
k_zscan(const float *__restrict__ dz, const float *z0, float *__restrict__ snapZ, float *z_out,
        int S)
{
    __shared__ float tot[8][D];
    const int f = threadIdx.x % D, g = threadIdx.x / D;
    const int64_t chain = blockIdx.x;
    const int per = (S + 7) / 8;
    const int s0 = g * per < S ? g * per : S, s1 = s0 + per < S ? s0 + per : S;
    const float *src = dz + chain * S * D + f;
    float t = 0.f;
#pragma unroll 8
    for (int s = s0; s < s1; ++s) t += src[(int64_t)s * D];
    float z = z0 ? z0[chain * D + f] : 0.f;
    tot[g][f] = t;
    __syncthreads();
    for (int j = 0; j < g; ++j) z += tot[j][f];
    float *dst = snapZ + chain * S * D + f;
    for (int s = s0; s < s1; ++s) {
        dst[(int64_t)s * D] = z;
        z += src[(int64_t)s * D];
    }
    if (g == 7) z_out[chain * D + f] = z;
}

// ---------------------------------------------------------------- per-segment increments

template <int D, bool DELTA>
struct IncrCfg {
    static_assert(D == 64 || D == 128, "tensor-core memory increments: d = 64 or 128");
    static constexpr int CH = 64;                    // tokens per chunk
    static constexpr int NB = D / 64;                // 64-column boxes of K, V and W
    static constexpr int BOX = CH * 128;             // 64 rows x 64 bf16 (128-byte rows)
    // ring slot (TMA): the K chunk, turned into sigma_hi in place (features padded to 128:
    // for d = 64 the second box stays zero), then the V chunk
    static constexpr int RS = 4;
    static constexpr int OFF_SH = 0;
    static constexpr int OFF_V = 2 * BOX;
    static constexpr int SLOT = (2 + NB) * BOX;
    // operand set (two, alternating by chunk): sigma_lo (bf16, padded like sigma_hi) and, for
    // the delta rule, sigma in f16 (padded the same way) and W' = 2^e sigma / den in f16
    static constexpr int OFF_SL = 0;
    static constexpr int OFF_S16 = 2 * BOX;
    static constexpr int OFF_W16 = 4 * BOX;
    static constexpr int OSET = DELTA ? (4 + NB) * BOX : 2 * BOX;
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_OPS = RS * SLOT;
    // additive rule: a K-major tile of ones (16 columns x 64 tokens), the B operand of
    // sigma(K)^T 1, which gives the segment's sum of sigma(k_t) beside B_s
    static constexpr int OFF_ONES = OFF_OPS + 2 * OSET;
    static constexpr int ONES = DELTA ? 0 : 16 * 128;
    static constexpr int OFF_BAR = OFF_ONES + ONES;
    static constexpr int NBAR = 3 * RS + 2 + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr int ACC = DELTA ? 2 * D : D;     // accumulator columns: B_s | A_s
    static constexpr int ZC = DELTA ? 0 : 32;         // additive rule: columns of sigma(K)^T 1
    static constexpr int T_Z = 2 * ACC;               // those of the two sets follow both B_s
    static constexpr uint32_t TMEM_COLS = 2 * (ACC + ZC) <= 256 ? 256 : 512;
    static constexpr int THREADS = 768;
    static constexpr int WORKERS = 512;              // 16 warps: eight threads per token row
    static constexpr int FPT = D / 8;                // features per worker thread: one 16-byte
                                                     // chunk of each 64-feature box
    static_assert(SLOT % 1024 == 0 && OSET % 1024 == 0, "operand tiles must be 1024-aligned");
    static_assert(ALLOC <= 232448, "shared memory");
};

struct IncrArgs {
    const float *snapZ;        // [chains * S, D]: z_{s-1} (delta)
    float *Bs;                 // [chains * S, D, D] fp32: sigma(K_s)^T V_s
    __nv_bfloat16 *Ahi, *Alo;  // [chains * S, D, D]: A_s split into two bf16 parts (delta)
    float *dz;                 // [chains * S, D]: sum of sigma(k_t) over segment s (additive)
    int64_t L;
    int N, S;
    int items;                 // chains * S
};

// The scale of W' for the item whose z_{s-1} is z: 2^e with Sigma_f z_f in [2^(e-1), 2^e)
// (e = 0 when the sum is 0).  Then den_t / 2^e is a z-weighted mean of sigma(k_t) within a
// factor 2, so W' = 2^e sigma / den is O(1) and fits f16; A_s = 2^-e sigma^T W'.  Workers
// and epilogue call this on the same z and get the same e (one fixed summation order).
__device__ __forceinline__ int incr_scale_exp(const float *z, int d)
{
    const float4 *z4 = reinterpret_cast<const float4 *>(z);
    float sum = 0.f;
    for (int i = 0; i < d / 4; ++i) {
        const float4 x = __ldg(z4 + i);
        sum = (((sum + x.x) + x.y) + x.z) + x.w;
    }
    if (!(sum > 0.f)) return 0;
    int e;
    frexpf(sum, &e);
    return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// Two floats to f16x2 (lo in the lower half), values past f16's range clamped to its largest
// finite value by the conversion itself
__device__ __forceinline__ uint32_t pack_f16x2_sat(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^e as a float (|e| <= 100)
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

enum : int { WI_EMPTY = 701, WI_FULL = 702, WI_OFREE = 703, WI_AREADY = 704, WI_ACCFREE = 705,
             WI_ACCFULL = 706, WI_DRAIN = 707 };

__device__ __forceinline__ void incr_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WI_DRAIN);
            return;
        }
    }
}

// Persistent: CTA b takes items (chain, segment) b, b + grid, ...; every role walks the same
// schedule of 64-token chunks, numbered g across the CTA's items.
//   warp 0       TMA producer: K and V chunks into a ring of RS slots, running ahead across
//                item boundaries
//   warp 1       MMA issuer: per chunk, B += sigma_hi^T V + sigma_lo^T V (bf16 operands) and,
//                for the delta rule, A' += sigma_f16^T W' (f16 operands), into the item's
//                accumulator set (two sets, alternating by item)
//   warps 4-19   workers: eight threads per token row turn K into sigma_hi (in place) and
//                sigma_lo and, for the delta rule, sigma in f16, den = sigma . z_{s-1} and
//                W' = 2^e sigma / den in f16 into the chunk's operand set (two sets,
//                alternating by chunk)
//   warps 20-23  epilogue: lane i of the item's accumulator is key feature i; row i of B_s
//                (fp32) and of A_s = 2^-e A' (bf16 hi, lo) to global memory, while the next
//                item's MMAs fill the other accumulator set
// Precision: B_s carries sigma to about 16 bits (hi + lo); A_s, which only scales the
// correction A_s M_{s-1}, carries sigma and W' to f16's 11 bits.
template <int D, bool DELTA>
__global__ void __launch_bounds__(768, 1)
k_mem_incr(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
           const IncrArgs a)
{
    using C = IncrCfg<D, DELTA>;
    constexpr int RS = C::RS;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *ring = smem + C::OFF_RING, *ops = smem + C::OFF_OPS;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars, *empty = bars + RS, *aready = bars + 2 * RS;
    uint64_t *ofree = bars + 3 * RS, *accfull = ofree + 2, *accfree = accfull + 2;
    uint64_t *mma_done = accfree + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < RS; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
            mbar_init(aready + i, C::WORKERS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(ofree + i, 1);
            mbar_init(accfull + i, 1);
            mbar_init(accfree + i, 128);
        }
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (D == 64) {  // the padded feature box of every sigma tile (hi, lo, f16) stays zero
        constexpr int NT = RS + (DELTA ? 4 : 2);
        for (int i = threadIdx.x; i < NT * (C::BOX / 16); i += blockDim.x) {
            const int t = i / (C::BOX / 16), o = i % (C::BOX / 16);
            uint8_t *base = t < RS ? ring + t * C::SLOT + C::OFF_SH
                                   : ops + ((t - RS) % 2) * C::OSET + ((t - RS) < 2 ? C::OFF_SL : C::OFF_S16);
            reinterpret_cast<uint4 *>(base + C::BOX)[o] = make_uint4(0, 0, 0, 0);
        }
    }
    if constexpr (!DELTA)
        for (int i = threadIdx.x; i < C::ONES / 16; i += blockDim.x)   // bf16 1.0 everywhere
            reinterpret_cast<uint4 *>(smem + C::OFF_ONES)[i] =
                make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t T = *tmem_holder;

    auto item_rows = [&](int item) {
        const int64_t row0 = (int64_t)(item % a.S) * a.N;
        return (int)(a.L - row0 < a.N ? a.L - row0 : a.N);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int g = 0, issued = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x) {
                const int chain = item / a.S, row0 = (item % a.S) * a.N;
                const int nch = (item_rows(item) + C::CH - 1) / C::CH;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int st = g % RS;
                    if (g >= RS && !(ok = mbar_wait_short(empty + st, ((g / RS) - 1) & 1, abort, WI_EMPTY)))
                        break;
                    uint8_t *slot = ring + st * C::SLOT;
                    mbar_arrive_expect_tx(full + st, (uint32_t)(2 * C::NB * C::BOX));
                    for (int b = 0; b < C::NB; ++b) {
                        tma_load_3d(slot + C::OFF_SH + b * C::BOX, &tmK, full + st, b * 64,
                                    row0 + c * C::CH, chain);
                        tma_load_3d(slot + C::OFF_V + b * C::BOX, &tmV, full + st, b * 64,
                                    row0 + c * C::CH, chain);
                    }
                    issued = g + 1;
                }
            }
            if (*abort)
                for (int h = (issued > RS ? issued - RS : 0); h < issued; ++h)
                    incr_drain(full + h % RS, (h / RS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t id = idesc_bf16(128, D, 1, 1);      // both operands MN-major
            constexpr uint32_t id16 = idesc_f16(128, D, 1, 1);
            constexpr uint32_t idZ = idesc_bf16(128, 16, 1, 0);     // sigma(K)^T 1, ones K-major
            const uint32_t aRing = smem_u32(ring), aOps = smem_u32(ops);
            const uint32_t aOnes = smem_u32(smem + C::OFF_ONES);
            int g = 0, j = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++j) {
                const int nch = (item_rows(item) + C::CH - 1) / C::CH;
                const uint32_t acc = T + (j & 1) * C::ACC;
                // the epilogue of item j - 2 has read this accumulator set
                if (j >= 2 && !(ok = mbar_wait_short(accfree + (j & 1), ((j >> 1) - 1) & 1, abort, WI_ACCFREE)))
                    break;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int st = g % RS;
                    if (!(ok = mbar_wait_short(aready + st, (g / RS) & 1, abort, WI_AREADY))) break;
                    tc_fence_after();
                    const uint32_t sl = aRing + st * C::SLOT, os = aOps + (g & 1) * C::OSET;
#pragma unroll
                    for (int kk = 0; kk < C::CH / 16; ++kk) {       // 16 tokens per step
                        const uint32_t k2 = kk * 2048;
                        const uint64_t ah = sdesc_sw128(sl + C::OFF_SH + k2, C::BOX, 1024);
                        const uint64_t al = sdesc_sw128(os + C::OFF_SL + k2, C::BOX, 1024);
                        const uint64_t bv = sdesc_sw128(sl + C::OFF_V + k2, C::BOX, 1024);
                        const uint32_t first = (c > 0 || kk > 0) ? 1u : 0u;
                        mma_ss(acc, ah, bv, id, first);
                        mma_ss(acc, al, bv, id, 1u);
                        if constexpr (!DELTA) {      // every element of the tile is 1: any K offset
                            const uint64_t b1 = sdesc_sw128(aOnes + kk * 32, 16, 1024);
                            const uint32_t accz = T + C::T_Z + (j & 1) * C::ZC;
                            mma_ss(accz, ah, b1, idZ, first);
                            mma_ss(accz, al, b1, idZ, 1u);
                        }
                        if constexpr (DELTA) {
                            const uint64_t a16 = sdesc_sw128(os + C::OFF_S16 + k2, C::BOX, 1024);
                            const uint64_t bw = sdesc_sw128(os + C::OFF_W16 + k2, C::BOX, 1024);
                            mma_ss(acc + D, a16, bw, id16, first);
                        }
                    }
                    mma_commit(empty + st);
                    mma_commit(ofree + (g & 1));
                }
                if (ok) mma_commit(accfull + (j & 1));
            }
            mma_commit(mma_done);
            incr_drain(mma_done, 0);
        }
    } else if (warp >= 4 && warp < 20) {
        // ---------------------------------------------------------------- workers
        const int w = threadIdx.x - 128;            // 0..511
        // token row of the chunk; the thread's 16-byte chunk q of every 64-feature box
        // (features 64 i + 8 q + e), so the eight threads of a row cover its 128 bytes per box
        const int t = w >> 3, q = w & 7;
        constexpr int CPT = C::NB;                  // 16-byte chunks per thread
        const uint64_t one2 = f2_pack(1.f, 1.f);
        const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
        int g = 0, j = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++j) {
            const int rows = item_rows(item);
            const int nch = (rows + C::CH - 1) / C::CH;
            // z_{s-1} at this thread's features (no block-wide barrier: a worker that gives up
            // on a wait must not leave the others waiting at one)
            float zr[C::FPT];
            float wscale = 1.f;
            if constexpr (DELTA) {
                wscale = pow2f(incr_scale_exp(a.snapZ + (int64_t)item * D, D));
                const float *zi = a.snapZ + (int64_t)item * D + 8 * q;
#pragma unroll
                for (int e = 0; e < C::FPT / 4; ++e) {
                    const float4 x = __ldg(reinterpret_cast<const float4 *>(zi + (e >> 1) * 64) + (e & 1));
                    zr[4 * e] = x.x;
                    zr[4 * e + 1] = x.y;
                    zr[4 * e + 2] = x.z;
                    zr[4 * e + 3] = x.w;
                }
            }
            for (int c = 0; c < nch; ++c, ++g) {
                const int st = g % RS;
                if (!(ok = mbar_wait(full + st, (g / RS) & 1, abort, WI_FULL))) break;
                if (g >= 2 && !(ok = mbar_wait(ofree + (g & 1), ((g >> 1) - 1) & 1, abort, WI_OFREE)))
                    break;
                uint8_t *slot = ring + st * C::SLOT, *os = ops + (g & 1) * C::OSET;
                // rows past the head's L (zero-filled by TMA) carry sigma = 0 (only a chunk
                // that reaches past L needs the mask)
                const bool partial = c * C::CH + C::CH > rows;
                const uint32_t keep = c * C::CH + t < rows ? 0xFFFFFFFFu : 0u;
                float sg[C::FPT];
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int off = i * C::BOX + t * 128 + ((q ^ (t & 7)) << 4);
                    uint4 *ph = reinterpret_cast<uint4 *>(slot + C::OFF_SH + off);
                    const uint4 v = *ph;
                    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                    uint32_t hi[4], lo[4], h16[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // sigma = max(x + 1, e^min(x, 0)) on packed fp32 pairs (as elu1)
                        const float x0 = __uint_as_float(in[e] << 16), x1 = __uint_as_float(in[e] & 0xffff0000u);
                        float a0, a1, p0, p1;
                        f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
                        f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
                        float s0 = fmaxf(p0, ex2(a0)), s1 = fmaxf(p1, ex2(a1));
                        if (partial) {
                            s0 = __uint_as_float(__float_as_uint(s0) & keep);
                            s1 = __uint_as_float(__float_as_uint(s1) & keep);
                        }
                        sg[i * 8 + 2 * e] = s0;
                        sg[i * 8 + 2 * e + 1] = s1;
                        hi[e] = pack_bf16x2(s0, s1);
                        float l0, l1;
                        f2_unpack(f2_sub(f2_pack(s0, s1), f2_pack(__uint_as_float(hi[e] << 16),
                                                                  __uint_as_float(hi[e] & 0xffff0000u))),
                                  l0, l1);
                        lo[e] = pack_bf16x2(l0, l1);
                        if constexpr (DELTA) h16[e] = pack_f16x2(s0, s1);
                    }
                    *ph = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(os + C::OFF_SL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    if constexpr (DELTA)
                        *reinterpret_cast<uint4 *>(os + C::OFF_S16 + off) = make_uint4(h16[0], h16[1], h16[2], h16[3]);
                }
                if constexpr (DELTA) {
                    uint64_t dp2[2] = {0ull, 0ull};
#pragma unroll
                    for (int e = 0; e < C::FPT / 2; ++e)
                        dp2[e & 1] = f2_fma(f2_pack(sg[2 * e], sg[2 * e + 1]), f2_pack(zr[2 * e], zr[2 * e + 1]),
                                            dp2[e & 1]);
                    float d0, d1, d2, d3;
                    f2_unpack(dp2[0], d0, d1);
                    f2_unpack(dp2[1], d2, d3);
                    float den = (d0 + d1) + (d2 + d3);
                    den += __shfl_xor_sync(0xffffffffu, den, 1);
                    den += __shfl_xor_sync(0xffffffffu, den, 2);
                    den += __shfl_xor_sync(0xffffffffu, den, 4);
                    const float inv = den == 0.f ? 0.f : wscale / den;
                    const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
                    for (int i = 0; i < CPT; ++i) {
                        const int off = i * C::BOX + t * 128 + ((q ^ (t & 7)) << 4);
                        uint32_t w16[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {   // W' >= 0; clamped to f16's largest finite value
                            float w0, w1;
                            f2_unpack(f2_mul(f2_pack(sg[i * 8 + 2 * e], sg[i * 8 + 2 * e + 1]), inv2), w0, w1);
                            w16[e] = pack_f16x2_sat(w0, w1);
                        }
                        *reinterpret_cast<uint4 *>(os + C::OFF_W16 + off) = make_uint4(w16[0], w16[1], w16[2], w16[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(aready + st);
            }
        }
    } else if (warp >= 20) {
        // ---------------------------------------------------------------- epilogue
        const int i = (warp & 3) * 32 + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool live = D == 128 || (warp & 3) < 2;      // lanes past d hold nothing
        int j = 0;
        for (int item = blockIdx.x; item < a.items; item += gridDim.x, ++j) {
            if (!mbar_wait(accfull + (j & 1), (j >> 1) & 1, abort, WI_ACCFULL)) break;
            tc_fence_after();
            const uint32_t acc = T + (j & 1) * C::ACC;
            const float ascale = DELTA ? pow2f(-incr_scale_exp(a.snapZ + (int64_t)item * D, D)) : 1.f;
            if (live) {
#pragma unroll 1
                for (int c0 = 0; c0 < C::ACC; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + acc + c0, r);
                    tmem_ld_wait();
                    const int col = c0 % D;
                    const int64_t o = ((int64_t)item * D + i) * D + col;
                    if (c0 < D) {
                        float4 *dst = reinterpret_cast<float4 *>(a.Bs + o);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                                 __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
                    } else {
                        uint32_t hi[16], lo[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float x0 = __uint_as_float(r[2 * e]) * ascale;
                            const float x1 = __uint_as_float(r[2 * e + 1]) * ascale;
                            const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                            hi[e] = *reinterpret_cast<const uint32_t *>(&h);
                            lo[e] = pack_bf16x2(x0 - __low2float(h), x1 - __high2float(h));
                        }
                        uint4 *dh = reinterpret_cast<uint4 *>(a.Ahi + o);
                        uint4 *dl = reinterpret_cast<uint4 *>(a.Alo + o);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            dh[e] = make_uint4(hi[4 * e], hi[4 * e + 1], hi[4 * e + 2], hi[4 * e + 3]);
                            dl[e] = make_uint4(lo[4 * e], lo[4 * e + 1], lo[4 * e + 2], lo[4 * e + 3]);
                        }
                    }
                }
                if constexpr (!DELTA) {          // every column holds the same sum
                    uint32_t r[16];
                    tmem_ld16(lane_base + T + C::T_Z + (j & 1) * C::ZC, r);
                    tmem_ld_wait();
                    a.dz[(int64_t)item * D + i] = __uint_as_float(r[0]);
                }
            }
            tc_fence_before();
            mbar_arrive(accfree + (j & 1));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(T, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- the serial parts

// Additive rule: M_{s-1} = M0 + sum_{j<s} B_j, writing the snapshot of every M_{s-1} (bf16
// and / or fp32) and M_out.  A block covers 256 / CH groups of 4 consecutive elements of a
// chain's M with CH threads each: thread c sums B_j over its chunk of consecutive segments,
// the chunk totals give every chunk its starting value, and the thread then walks its chunk
// writing the snapshots (the summation order is fixed by the chunking).  Every thread reads
// its elements of M0 before the block barrier and only the last chunk's thread writes
// M_out, so M0 and M_out may alias.  CH = 1 (few segments) is a single walk.
template <int D, int CH>
__global__ void __launch_bounds__(256)
k_mem_prefix(const float *__restrict__ Bs, const float *M0, __nv_bfloat16 *__restrict__ snapMb,
             float *M_out, int S, int64_t chains, float *__restrict__ snapMf = nullptr)
{
    constexpr int64_t E4 = (int64_t)D * D / 4;
    constexpr int COLS = 256 / CH;
    __shared__ float4 tot[CH][COLS];
    const int col = threadIdx.x % COLS, c = threadIdx.x / COLS;
    const int64_t i = blockIdx.x * (int64_t)COLS + col;
    const bool live = i < chains * E4;
    const int64_t chain = live ? i / E4 : 0, e = i % E4;
    const int len = (S + CH - 1) / CH;
    const int s0 = c * len, s1 = s0 + len < S ? s0 + len : S;
    const float4 *b = reinterpret_cast<const float4 *>(Bs) + chain * S * E4 + e;
    float4 m = make_float4(0.f, 0.f, 0.f, 0.f), t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) {
        if (M0) m = reinterpret_cast<const float4 *>(M0)[i];
#pragma unroll 4
        for (int s = s0; CH > 1 && s < s1; ++s) {
            const float4 x = b[(int64_t)s * E4];
            t.x += x.x;
            t.y += x.y;
            t.z += x.z;
            t.w += x.w;
        }
    }
    tot[c][col] = t;
    __syncthreads();
    if (!live) return;
    for (int j = 0; j < c; ++j) {
        const float4 x = tot[j][col];
        m.x += x.x;
        m.y += x.y;
        m.z += x.z;
        m.w += x.w;
    }
    uint2 *snap = snapMb ? reinterpret_cast<uint2 *>(snapMb) + chain * S * E4 + e : nullptr;
    float4 *snapf = snapMf ? reinterpret_cast<float4 *>(snapMf) + chain * S * E4 + e : nullptr;
#pragma unroll 4
    for (int s = s0; s < s1; ++s) {
        if (snap) snap[(int64_t)s * E4] = make_uint2(pack_bf16x2(m.x, m.y), pack_bf16x2(m.z, m.w));
        if (snapf) snapf[(int64_t)s * E4] = m;
        const float4 x = b[(int64_t)s * E4];
        m.x += x.x;
        m.y += x.y;
        m.z += x.z;
        m.w += x.w;
    }
    if (c == CH - 1) reinterpret_cast<float4 *>(M_out)[i] = m;
}

template <int D>
struct MChainCfg {
    static_assert(D == 64 || D == 128, "tensor-core delta recurrence: d = 64 or 128");
    static constexpr int CB = 16;                   // value columns per CTA
    static constexpr int THREADS = 384;             // TMA, MMA, 2 idle, 8 update warps
    static constexpr int NK = D / 64;               // 64-wide boxes along the contraction
    static constexpr int ABOX = 128 * 128;          // 128 rows x 64 bf16
    static constexpr int ATILE = NK * ABOX;         // A_hi (or A_lo) of one segment
    static constexpr int ST = 3;                    // A_s loads run this many segments ahead
    // per 64-wide box along the contraction, K-major: rows 0..CB-1 M^T hi, rows CB..2CB-1
    // M^T lo, so one N = 2 CB product takes A_hi against both parts
    static constexpr int BBOX = 2 * CB * 128;
    static constexpr int BTILE = NK * BBOX;
    static_assert(CB % 8 == 0, "the lo rows keep the hi rows' swizzle phase");
    static constexpr int OFF_A = 0;                 // per stage: A_hi | A_lo
    static constexpr int OFF_B = ST * 2 * ATILE;    // [M^T hi ; M^T lo] per box
    static constexpr int OFF_BAR = OFF_B + BTILE;
    static constexpr int NBAR = 2 * ST + 3;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(OFF_B % 1024 == 0 && BTILE % 1024 == 0, "operand tiles must be 1024-aligned");
    static_assert(ALLOC <= 232448, "shared memory");
};

struct MChainArgs {
    const float *M0;           // may be NULL (zeros); may alias M_out exactly
    const float *Bs;           // [chains * S, D, D]
    __nv_bfloat16 *snapMb;     // [chains * S, D, D]: bf16 M_{s-1}, or NULL
    float *snapMf;             // [chains * S, D, D]: fp32 M_{s-1}, or NULL
    float *M_out;
    int S;
    int reverse;               // walk the segments from the last to the first
};

// 32 lanes x 8 consecutive 32-bit columns (warp-uniform address): thread t gets lane base + t
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

enum : int { WM_A_EMPTY = 801, WM_B = 802, WM_A_FULL = 803, WM_D = 804, WM_DRAIN = 805 };

__device__ __forceinline__ void mchain_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WM_DRAIN);
            return;
        }
    }
}

// Delta rule: M_s = M_{s-1} + B_s - A_s M_{s-1} in segment order (with `reverse`, from the
// last segment to the first: the backward's dM_{s-1} = dM_s + G_s - A_s dM_s, A_s being
// symmetric; the snapshot of each step is then the gradient after the segment).  One CTA per (chain, 16
// value columns); column block j of M_s needs only column block j of M_{s-1}.  Warp 0: TMA
// of A_s (hi and lo parts, K-major, two stages ahead).  Warp 1: MMA issuer, per 16-wide step
// of the contraction A_hi [M_hi | M_lo] (one N = 32 product into 32 TMEM columns) and A_lo M_hi
// into the first 16; the threads add the two halves: D = A_hi M_hi + A_lo M_hi + A_hi M_lo.
// Warps 4-11: two threads per row i of the block, eight columns each, in fp32 registers;
// each writes its part of the M^T hi / lo operand, signals the issuer, then (while the
// products run) stores the snapshot and loads B_s, and applies M += B_s - D.  d = 64 runs
// as 128 rows with zero rows 64..127 of A.
template <int D>
__global__ void __launch_bounds__(384, 1)
k_mem_chain(const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
            const MChainArgs a)
{
    using C = MChainCfg<D>;
    constexpr int ST = C::ST, CB = C::CB;
    constexpr int NBLK = D / CB;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int64_t chain = blockIdx.x / NBLK;
    const int cb = (blockIdx.x % NBLK) * CB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *a_full = bars, *a_empty = bars + ST, *b_ready = bars + 2 * ST, *d_full = b_ready + 1;
    uint64_t *mma_done = d_full + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(a_full + i, 1);
            mbar_init(a_empty + i, 1);
        }
        mbar_init(b_ready, 256);
        mbar_init(d_full, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (D == 64)   // rows 64..127 of every A tile stay zero (the loads fill rows 0..63)
        for (int i = threadIdx.x; i < ST * 2 * (C::ABOX / 32); i += blockDim.x) {
            const int t = i / (C::ABOX / 32), o = i % (C::ABOX / 32);
            reinterpret_cast<uint4 *>(smem + C::OFF_A + t * C::ATILE + C::ABOX / 2)[o] =
                make_uint4(0, 0, 0, 0);
        }
    if (warp == 1) tmem_alloc(tmem_holder, 32);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t T = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmAh);
            prefetch_tmap(&tmAl);
            int issued = 0;
            for (int s = 0; s < a.S; ++s) {
                const int st = s % ST;
                if (s >= ST && !mbar_wait_short(a_empty + st, ((s / ST) - 1) & 1, abort, WM_A_EMPTY))
                    break;
                uint8_t *dst = smem + C::OFF_A + st * 2 * C::ATILE;
                const int slot = (int)(chain * a.S + (a.reverse ? a.S - 1 - s : s));
                mbar_arrive_expect_tx(a_full + st, (uint32_t)(2 * C::NK * D * 128));
                for (int b = 0; b < C::NK; ++b) {
                    tma_load_3d(dst + b * C::ABOX, &tmAh, a_full + st, b * 64, 0, slot);
                    tma_load_3d(dst + C::ATILE + b * C::ABOX, &tmAl, a_full + st, b * 64, 0, slot);
                }
                issued = s + 1;
            }
            if (*abort)
                for (int s = (issued > ST ? issued - ST : 0); s < issued; ++s)
                    mchain_drain(a_full + s % ST, (s / ST) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // columns 0..CB-1: A_hi M_hi + A_lo M_hi; columns CB..2CB-1: A_hi M_lo
            constexpr uint32_t id2 = idesc_bf16(128, 2 * CB, 0, 0);
            constexpr uint32_t id1 = idesc_bf16(128, CB, 0, 0);
            // descriptors of the tiles' bases; an offset (a multiple of 16 bytes inside shared
            // memory) adds to the address field without carrying out of it
            const uint64_t dA = sdesc_sw128(smem_u32(smem + C::OFF_A), 16, 1024);
            const uint64_t dB = sdesc_sw128(smem_u32(smem + C::OFF_B), 16, 1024);
            for (int s = 0; s < a.S; ++s) {
                const int st = s % ST;
                if (!mbar_wait_short(b_ready, s & 1, abort, WM_B)) break;
                if (!mbar_wait_short(a_full + st, (s / ST) & 1, abort, WM_A_FULL)) break;
                tc_fence_after();
                const uint32_t ah = st * 2 * C::ATILE, al = ah + C::ATILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ao = (kk >> 2) * C::ABOX + (kk & 3) * 32;
                    const uint64_t db = dB + (((kk >> 2) * C::BBOX + (kk & 3) * 32) >> 4);
                    mma_ss(T, dA + ((ah + ao) >> 4), db, id2, kk > 0 ? 1u : 0u);
                    mma_ss(T, dA + ((al + ao) >> 4), db, id1, 1u);
                }
                mma_commit(a_empty + st);
                mma_commit(d_full);
            }
            mma_commit(mma_done);
            mchain_drain(mma_done, 0);
        }
    } else if (warp >= 4) {
        const int i = (threadIdx.x - 128) & 127;    // row of M (key feature), TMEM lane
        constexpr int CH = CB / 2;                  // two threads per row, CH columns each
        const int c0 = ((threadIdx.x - 128) >> 7) * CH;
        const bool live = i < D;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint8_t *sB = smem + C::OFF_B;
        float m[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) m[j] = 0.f;
        if (live && a.M0) {
            const float4 *src = reinterpret_cast<const float4 *>(a.M0 + (chain * D + i) * D + cb + c0);
#pragma unroll
            for (int e = 0; e < CH / 4; ++e) {
                const float4 x = src[e];
                m[4 * e] = x.x;
                m[4 * e + 1] = x.y;
                m[4 * e + 2] = x.z;
                m[4 * e + 3] = x.w;
            }
        }
        // element (j, k = i) of a K-major [CB rows x D] tile
        const int kb = i >> 6, kc = i & 63;
        bool ok = true;
        for (int s = 0; s < a.S; ++s) {
            const int64_t slot = chain * a.S + (a.reverse ? a.S - 1 - s : s);
            if (live) {
#pragma unroll
                for (int jj = 0; jj < CH; ++jj) {
                    const int j = c0 + jj;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(m[jj]);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(m[jj] - __bfloat162float(hi));
                    const int o = kb * C::BBOX + j * 128 + ((((kc >> 3) ^ (j & 7))) << 4) + (kc & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16 *>(sB + o) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sB + CB * 128 + o) = lo;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_ready);
            // off the serial path, while the products run: the snapshot M_{s-1} and B_s
            float4 bs[CH / 4];
            if (live) {
                if (a.snapMb) {
                    uint32_t pk[CH / 2];
#pragma unroll
                    for (int e = 0; e < CH / 2; ++e) pk[e] = pack_bf16x2(m[2 * e], m[2 * e + 1]);
                    uint4 *dst = reinterpret_cast<uint4 *>(a.snapMb + (slot * D + i) * D + cb + c0);
#pragma unroll
                    for (int e = 0; e < CH / 8; ++e)
                        dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
                if (a.snapMf) {
                    float4 *dst = reinterpret_cast<float4 *>(a.snapMf + (slot * D + i) * D + cb + c0);
#pragma unroll
                    for (int e = 0; e < CH / 4; ++e)
                        dst[e] = make_float4(m[4 * e], m[4 * e + 1], m[4 * e + 2], m[4 * e + 3]);
                }
                const float4 *src = reinterpret_cast<const float4 *>(a.Bs + (slot * D + i) * D + cb + c0);
#pragma unroll
                for (int e = 0; e < CH / 4; ++e) bs[e] = src[e];
            }
            // on the serial path: probe without the suspend hint
            if (!(ok = mbar_wait_short(d_full, s & 1, abort, WM_D))) break;
            tc_fence_after();
            // this thread's columns of both halves (c0 is uniform across the warp)
            uint32_t r0[CH], r1[CH];
            static_assert(CH == 8, "one tmem_ld8 per half");
            tmem_ld8(lane_base + T + c0, r0);
            tmem_ld8(lane_base + T + CB + c0, r1);
            tmem_ld_wait();
            if (live) {
#pragma unroll
                for (int e = 0; e < CH / 4; ++e) {
                    const uint32_t *d0 = r0 + 4 * e, *d1 = r1 + 4 * e;
                    m[4 * e] += bs[e].x - (__uint_as_float(d0[0]) + __uint_as_float(d1[0]));
                    m[4 * e + 1] += bs[e].y - (__uint_as_float(d0[1]) + __uint_as_float(d1[1]));
                    m[4 * e + 2] += bs[e].z - (__uint_as_float(d0[2]) + __uint_as_float(d1[2]));
                    m[4 * e + 3] += bs[e].w - (__uint_as_float(d0[3]) + __uint_as_float(d1[3]));
                }
            }
            tc_fence_before();
        }
        if (ok && live) {
            float4 *dst = reinterpret_cast<float4 *>(a.M_out + (chain * D + i) * D + cb + c0);
#pragma unroll
            for (int e = 0; e < CH / 4; ++e)
                dst[e] = make_float4(m[4 * e], m[4 * e + 1], m[4 * e + 2], m[4 * e + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(T, 32);
    }
}

}  // namespace tc
}  // namespace infini
