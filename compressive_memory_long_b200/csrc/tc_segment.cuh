// Fused Infini-attention segment kernel on the 5th-generation tensor cores (sm_100a).
//
// One CTA computes 128 query rows of one (batch b, query head h, segment s):
//   A_dot = causal softmax(Q K_s^T / sqrt(d)) V_s over keys of segment s up to the diagonal
//   A_mem = sigma(Q) M_{s-1} / (sigma(Q) . z_{s-1})        (0 where the denominator is 0)
//   out   = g A_mem + (1 - g) A_dot,  g = sigmoid(beta[h])
// (AI Wiki "Infini-Attention", "What happens inside the Infini-attention block?").
// With 64-token segments (N = 64) the 128 rows are two consecutive segments s, s + 1: one
// key step over the same 128 rows under a block-diagonal causal mask (each segment sees only
// its own keys), and two retrievals, sigma(Q) M_{s-1} into S0 for the first 64 rows and
// sigma(Q) M_s into S1 (unused by the single key step) for the others; the second snapshot
// is loaded into the key ring's second slot, which the single key step leaves free.
//
// Roles (256 threads):
//   warp 0      TMA producer: Q tile, M_{s-1} (bf16 snapshot), K/V tiles through a ring
//               of STAGES shared-memory slots (SWIZZLE_128B boxes of 128 rows x 64 cols).
//   warp 1      tcgen05.mma issuer (one thread): S_j = Q K_j^T into a double-buffered TMEM
//               tile, O += P_j V_j with P read from TMEM, and at the end R = sigma(Q) M.
//   warps 4-7   softmax / epilogue: thread r owns query row r (TMEM lane r).  Online
//               softmax with exp2, lazy rescaling (O is rescaled only when a row maximum
//               grows by more than 2^8), P rounded to bf16 and stored into TMEM; then
//               sigma(Q) written over Q in shared memory for the retrieval contraction, and
//               the gated output stored from registers.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,256+d) P0 [384,448) P1 [448,512);
// the retrieval result reuses S0.
// Every wait is bounded (tc_common.cuh): a wait that gives up records its id in
// g_wait_status and the CTA winds down without touching the outputs it did not finish.
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

template <int D>
struct SegCfg {
    static_assert(D == 64 || D == 128, "tensor-core segment kernel: d = 64 or 128");
    static constexpr int BQ = 128, BK = 128;
    static constexpr int STAGES = (D == 128) ? 2 : 3;
    static constexpr int TILE = 128 * D * 2;        // bytes of one 128-row bf16 tile
    static constexpr int BOX = 128 * 128;           // bytes of one 128-row x 64-col box
    static constexpr int MBYTES = D * D * 2;        // bf16 M_{s-1}
    static constexpr int MBOX = D * 128;            // bytes of one D-row x 64-col box of M
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE;
    static constexpr int OFF_V = OFF_K + STAGES * TILE;
    static constexpr int OFF_M = OFF_V + STAGES * TILE;
    static constexpr int OFF_Z = OFF_M + MBYTES;
    static constexpr int NBAR = 2 + 3 * STAGES + 2 + 2 + 4;
    static constexpr int OFF_BAR = OFF_Z + 2 * D * 4;   // z of one segment (two at N = 64)
    static_assert(STAGES >= 2 && MBYTES <= TILE, "second snapshot in the key ring's slot 1");
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;      // slack to align the base to 1024 B
};

struct SegArgs {
    const float *beta;
    const float *snapZ;    // [chains * S, D] fp32 z_{s-1}
    __nv_bfloat16 *out;    // [B, H, L, D]
    int64_t L;             // rows per head; the last of the S segments may end before N rows
    int N, S, H, Hkv;
};

// wait ids recorded in g_wait_status
enum : int { W_KV_EMPTY = 101, W_Q = 102, W_K = 103, W_P = 104, W_V = 105, W_S = 106,
             W_PV = 107, W_PV_LAST = 108, W_R = 109, W_M = 110, W_SQ = 111, W_DRAIN = 112 };

// Wait without the abort shortcut: used when winding down, so that nothing a CTA issued
// (TMA copies, MMAs) is still in flight when it exits.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, W_DRAIN);
            return;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(256, 1)
k_segment_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
             const SegArgs a)
{
    using C = SegCfg<D>;
    constexpr int ST = C::STAGES;
    // an earlier wait gave up: do nothing until it is read (one CTA-wide decision)
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    // N = 64: a CTA per pair of segments (s, s + 1); s1 = -1 when the pair has no second
    const bool pair = a.N == 64;
    int64_t bid = blockIdx.x;
    int qt, s, s1 = -1;
    if (pair) {
        const int U = (a.S + 1) / 2;
        s = 2 * (int)(bid % U);
        bid /= U;
        qt = 0;
        if (s + 1 < a.S) s1 = s + 1;
    } else {
        const int qtiles = a.N / C::BQ;
        qt = qtiles - 1 - (int)(bid % qtiles);   // longest rows first
        bid /= qtiles;
        s = (int)(bid % a.S);
        bid /= a.S;
    }
    // a last segment shorter than N: tiles past the head's L rows have nothing to do
    if ((int64_t)s * a.N + qt * C::BQ >= a.L) return;
    const int64_t bh = bid;
    const int h = (int)(bh % a.H);
    const int64_t b = bh / a.H;
    const int64_t chain = b * a.Hkv + h / (a.H / a.Hkv);
    const int nkv = qt + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sM = smem + C::OFF_M;
    float *sZ = reinterpret_cast<float *>(smem + C::OFF_Z);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars, *m_full = bars + 1;
    uint64_t *k_full = bars + 2, *v_full = k_full + ST, *kv_empty = v_full + ST;
    uint64_t *s_full = kv_empty + ST, *p_full = s_full + 2;
    uint64_t *pv_done = p_full + 2, *sq_full = pv_done + 1, *r_full = sq_full + 1;
    uint64_t *mma_done = r_full + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(m_full, 1);
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
        }
        mbar_init(pv_done, 1);
        mbar_init(sq_full, 128);
        mbar_init(r_full, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_S0 = tmem, T_S1 = tmem + 128, T_O = tmem + 256;
    const uint32_t T_P0 = tmem + 384, T_P1 = tmem + 448;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmM);
            const int q_row = s * a.N + qt * C::BQ;
            const int kv_row0 = s * a.N;
            mbar_arrive_expect_tx(q_full, C::TILE);
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sQ + cb * C::BOX, &tmQ, q_full, cb * 64, q_row, (int)bh);
            mbar_arrive_expect_tx(m_full, (s1 >= 0 ? 2 : 1) * C::MBYTES);
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sM + cb * C::MBOX, &tmM, m_full, cb * 64, 0, (int)(chain * a.S + s));
            if (s1 >= 0)
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sK + C::TILE + cb * C::MBOX, &tmM, m_full, cb * 64, 0,
                                (int)(chain * a.S + s1));
            int issued = 0;
            for (int j = 0; j < nkv; ++j) {
                const int st = j % ST;
                if (j >= ST && !mbar_wait(kv_empty + st, ((j / ST) - 1) & 1, abort, W_KV_EMPTY))
                    break;
                mbar_arrive_expect_tx(k_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sK + st * C::TILE + cb * C::BOX, &tmK, k_full + st, cb * 64,
                                kv_row0 + j * C::BK, (int)chain);
                mbar_arrive_expect_tx(v_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sV + st * C::TILE + cb * C::BOX, &tmV, v_full + st, cb * 64,
                                kv_row0 + j * C::BK, (int)chain);
                issued = j + 1;
            }
            if (*abort) {   // let every copy still in flight land before the CTA exits
                mbar_drain(q_full, 0);
                mbar_drain(m_full, 0);
                for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j) {
                    mbar_drain(k_full + j % ST, (j / ST) & 1);
                    mbar_drain(v_full + j % ST, (j / ST) & 1);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);     // P/sigma(Q) x V/M (MN-major)
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            const uint32_t aM = smem_u32(sM);
            bool ok = mbar_wait(q_full, 0, abort, W_Q);

            auto issue_pv = [&](int i) -> bool {
                if (!mbar_wait(p_full + (i & 1), (i >> 1) & 1, abort, W_P)) return false;
                if (!mbar_wait(v_full + i % ST, (i / ST) & 1, abort, W_V)) return false;
                tc_fence_after();
                const uint32_t tP = (i & 1) ? T_P1 : T_P0;
                const uint32_t vbase = aV + (i % ST) * C::TILE;
#pragma unroll
                for (int kk = 0; kk < C::BK / 16; ++kk) {
                    const uint64_t bd = sdesc_sw128(vbase + kk * 2048, C::BOX, 1024);
                    mma_ts(T_O, tP + kk * 8, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(pv_done);
                mma_commit(kv_empty + i % ST);
                return true;
            };

            for (int j = 0; ok && j < nkv; ++j) {
                const int st = j % ST;
                if (!(ok = mbar_wait(k_full + st, (j / ST) & 1, abort, W_K))) break;
                tc_fence_after();
                const uint32_t dS = (j & 1) ? T_S1 : T_S0;
                const uint32_t kbase = aK + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(dS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + (j & 1));
                if (j > 0) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(nkv - 1);
            // retrieval R = sigma(Q) M_{s-1} into S0 (and sigma(Q) M_s into S1 for a pair)
            if (ok) ok = mbar_wait(m_full, 0, abort, W_M);
            if (ok) ok = mbar_wait(sq_full, 0, abort, W_SQ);
            if (ok) {
                tc_fence_after();
                for (int x = 0; x < (s1 >= 0 ? 2 : 1); ++x) {
                    const uint32_t mb = x == 0 ? aM : aK + C::TILE;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(x == 0 ? T_S0 : T_S1, sdesc_sw128(aQ + off, 16, 1024),
                               sdesc_sw128(mb + kk * 2048, C::MBOX, 1024), idO, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(r_full);
            }
            // every MMA issued above completes before the CTA releases TMEM
            mma_commit(mma_done);
            mbar_drain(mma_done, 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- softmax / epilogue
        const int r = threadIdx.x - 128;                 // query row of this thread
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        const float *zsrc = a.snapZ + (chain * a.S + s) * (int64_t)D;
        for (int i = r; i < D; i += 128) {
            sZ[i] = zsrc[i];
            if (pair) sZ[D + i] = s1 >= 0 ? zsrc[D + i] : 0.f;   // z_s of the pair's second
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // the rows of a pair's second segment use its own memory (S1, z_s)
        const bool second = pair && r >= 64;
        const float *zr = sZ + (second ? D : 0);
        const int lo = second ? 64 : 0;                      // the first key this row may see

        const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            if (!(ok = mbar_wait(s_full + (j & 1), (j >> 1) & 1, abort, W_S))) break;
            tc_fence_after();
            const uint32_t tS = lane_base + ((j & 1) ? T_S1 : T_S0);
            uint32_t raw[4][32];
            tmem_ld32(tS + 0, raw[0]);
            tmem_ld32(tS + 32, raw[1]);
            tmem_ld32(tS + 64, raw[2]);
            tmem_ld32(tS + 96, raw[3]);
            tmem_ld_wait();
            if (j == qt) {                                  // causal mask on the diagonal tile
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > r || c < lo) raw[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            float pm[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pm[u] = __uint_as_float(raw[0][u]);
#pragma unroll
            for (int c = 8; c < 128; ++c) pm[c & 7] = fmaxf(pm[c & 7], __uint_as_float(raw[c >> 5][c & 31]));
            const float mt = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                   fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            // PV_{j-1} must be complete before O is rescaled or P is rewritten
            if (j > 0 && !(ok = mbar_wait(pv_done, (j - 1) & 1, abort, W_PV))) break;
            tc_fence_after();
            const bool resc = (mt - m_used) * kscale > 8.f;
            float alpha = 1.f;
            if (resc) {
                alpha = ex2((m_used - mt) * kscale);
                m_used = mt;
                l *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + T_O + c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(lane_base + T_O + c, o);
                }
            }
            const float mk = m_used * kscale;
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[2][32];
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                const float p0 = ex2(fmaf(__uint_as_float(raw[c >> 5][c & 31]), kscale, -mk));
                const float p1 = ex2(fmaf(__uint_as_float(raw[(c + 1) >> 5][(c + 1) & 31]), kscale, -mk));
                ps[(c >> 1) & 3] += p0 + p1;
                pk[c >> 6][(c >> 1) & 31] = pack_bf16x2(p0, p1);
            }
            l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
            const uint32_t tP = lane_base + ((j & 1) ? T_P1 : T_P0);
            tmem_st32(tP, pk[0]);
            tmem_st32(tP + 32, pk[1]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full + (j & 1));
        }
        if (ok) ok = mbar_wait(pv_done, (nkv - 1) & 1, abort, W_PV_LAST);
        if (ok) {
            tc_fence_after();
            // sigma(Q) over Q in shared memory (row r, swizzled chunks) and den = sigma(q) . z
            float den = 0.f;
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 *p = reinterpret_cast<uint4 *>(sQ + cb * C::BOX + r * 128 +
                                                         ((ch ^ (r & 7)) << 4));
                    uint4 v = *p;
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                        float x0 = __low2float(t), x1 = __high2float(t);
                        x0 = elu1(x0);
                        x1 = elu1(x1);
                        const int c = cb * 64 + ch * 8 + 2 * e;
                        den = fmaf(x0, zr[c], den);
                        den = fmaf(x1, zr[c + 1], den);
                        w[e] = pack_bf16x2(x0, x1);
                    }
                    *p = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(sq_full);
            if (mbar_wait(r_full, 0, abort, W_R)) {
                tc_fence_after();
                const float g = 1.f / (1.f + __expf(-a.beta[h]));
                const float wl = (1.f - g) / l;
                const float wm = den == 0.f ? 0.f : g / den;
                const int64_t row = (int64_t)s * a.N + (int64_t)qt * C::BQ + r;
                const bool live = row < a.L;                     // rows past L: not stored
                __nv_bfloat16 *orow = a.out + (bh * a.L + row) * D;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32], rr[32];
                    tmem_ld32(lane_base + T_O + c, o);
                    tmem_ld32(lane_base + (second ? T_S1 : T_S0) + c, rr);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float y0 = fmaf(__uint_as_float(rr[2 * e]), wm, __uint_as_float(o[2 * e]) * wl);
                        const float y1 = fmaf(__uint_as_float(rr[2 * e + 1]), wm, __uint_as_float(o[2 * e + 1]) * wl);
                        pk[e] = pack_bf16x2(y0, y1);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
                    if (live)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc
}  // namespace infini
