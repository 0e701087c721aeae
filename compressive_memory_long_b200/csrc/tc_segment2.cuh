// Fused Infini-attention segment kernel, two query tiles per CTA (sm_100a).
//
// Same arithmetic as tc_segment.cuh (AI Wiki "Infini-Attention", "What happens inside the
// Infini-attention block?"): per query row, causal softmax attention over the keys of its
// segment, the retrieval sigma(q) M_{s-1} / (sigma(q) . z_{s-1}) and the sigmoid gate.
//
// A CTA owns the query tiles A = 2p and B = 2p + 1 (128 rows each) of one (b, h, segment);
// both read the same K/V tiles, which are loaded once.  Tile B needs key tiles 0..2p+1,
// tile A 0..2p.  Two softmax warpgroups (A: warps 0-3, B: warps 4-7) work in ping-pong
// with the tensor core: while one warpgroup turns its S tile into P, the MMA thread
// (warp 9) runs the other tile's P V and Q K^T.  TMA producer: warp 8 (thread 0 issues the
// first loads right after the barriers exist, ahead of the TMEM allocation and the block
// barrier); warps 10-11 only lend their registers.
// The third warpgroup hands registers to the two softmax warpgroups (setmaxnreg), which
// hold a full 128-score row each.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+d), O_B [256+d, 256+2d).
// P (bf16) is written over the first 64 columns of its own S tile; S_X(j) is issued after
// PV_X(j-1) by the same thread, and tcgen05.mma operations execute in issue order, so P is
// read before the next S overwrites it.  Each S commit also covers the previous PV, so a
// warpgroup that sees S_X(j) may rescale O_X at once.  After the last PV the retrieval
// R_X = sigma(Q_X) M_{s-1} reuses S_X.  All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

template <int D>
struct Seg2Cfg {
    static_assert(D == 64 || D == 128, "tensor-core segment kernel: d = 64 or 128");
    static constexpr int THREADS = 384;
    // register split (setmaxnreg): launched at REGS per thread; the producer / MMA warpgroup
    // gives back to REGS_LOW, each softmax warpgroup grows to REGS_HIGH.  The three shares add
    // up exactly to the launch's THREADS * REGS.
    static constexpr int REGS = 168, REGS_LOW = 88, REGS_HIGH = 208;
    static_assert(128 * (2 * REGS_HIGH + REGS_LOW) == THREADS * REGS, "register split");
    static constexpr int STAGES = (D == 128) ? 2 : 3;
    static constexpr int TILE = 128 * D * 2;
    static constexpr int BOX = 128 * 128;
    static constexpr int MBYTES = D * D * 2;
    static constexpr int MBOX = D * 128;
    static constexpr int OFF_QA = 0;
    static constexpr int OFF_QB = TILE;
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + STAGES * TILE;
    static constexpr int OFF_M = OFF_V + STAGES * TILE;
    static constexpr int OFF_Z = OFF_M + MBYTES;
    static constexpr int NBAR = 2 + 3 * STAGES + 2 * 5 + 1;
    static constexpr int OFF_BAR = OFF_Z + D * 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
};

enum : int { W2_KV_EMPTY = 401, W2_Q = 402, W2_K = 403, W2_P = 404, W2_V = 405, W2_S = 406,
             W2_PV = 407, W2_R = 408, W2_M = 409, W2_SQ = 410, W2_DRAIN = 411 };

__device__ __forceinline__ void seg2_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, W2_DRAIN);
            return;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(384, 1)
k_segment_tc2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
              const SegArgs a)
{
    using C = Seg2Cfg<D>;
    constexpr int ST = C::STAGES;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int npairs = a.N / 256;
    int64_t bid = blockIdx.x;
    const int p = npairs - 1 - (int)(bid % npairs);     // heaviest pairs first
    bid /= npairs;
    const int s = (int)(bid % a.S);
    bid /= a.S;
    // a last segment shorter than N: tiles past the head's L rows have nothing to do
    if ((int64_t)s * a.N + p * 256 >= a.L) return;
    const int64_t bh = bid;
    const int h = (int)(bh % a.H);
    const int64_t b = bh / a.H;
    const int64_t chain = b * a.Hkv + h / (a.H / a.Hkv);
    const int nB = 2 * p + 2;                            // key tiles of tile B (A: nB - 1)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sQ[2] = {smem + C::OFF_QA, smem + C::OFF_QB};
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sM = smem + C::OFF_M;
    float *sZ = reinterpret_cast<float *>(smem + C::OFF_Z);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars, *m_full = bars + 1;
    uint64_t *k_full = bars + 2, *v_full = k_full + ST, *kv_empty = v_full + ST;
    uint64_t *s_full = kv_empty + ST, *p_full = s_full + 2, *pv_done = p_full + 2;
    uint64_t *sq_full = pv_done + 2, *r_full = sq_full + 2, *mma_done = r_full + 2;
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
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + x, 1);
            mbar_init(p_full + x, 128);
            mbar_init(pv_done + x, 1);
            mbar_init(sq_full + x, 128);
            mbar_init(r_full + x, 1);
        }
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
        // the first loads go out now, overlapping the TMEM allocation and the block barrier
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmM);
        mbar_arrive_expect_tx(q_full, 2 * C::TILE);
        for (int x = 0; x < 2; ++x)
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sQ[x] + cb * C::BOX, &tmQ, q_full, cb * 64, s * a.N + p * 256 + x * 128,
                            (int)bh);
        for (int j = 0; j < nB && j < ST; ++j) {
            mbar_arrive_expect_tx(k_full + j, C::TILE);
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sK + j * C::TILE + cb * C::BOX, &tmK, k_full + j, cb * 64,
                            s * a.N + j * 128, (int)chain);
            mbar_arrive_expect_tx(v_full + j, C::TILE);
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sV + j * C::TILE + cb * C::BOX, &tmV, v_full + j, cb * 64,
                            s * a.N + j * 128, (int)chain);
        }
        mbar_arrive_expect_tx(m_full, C::MBYTES);
        for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sM + cb * C::MBOX, &tmM, m_full, cb * 64, 0, (int)(chain * a.S + s));
    }
    if (warp == 9) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_S[2] = {tmem, tmem + 128};
    const uint32_t T_O[2] = {tmem + 256, tmem + 256 + D};

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LOW));
      if (warp == 8) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            // Q, M and the first ST key / value tiles were issued by thread 0
            const int kv_row0 = s * a.N;
            int issued = nB < ST ? nB : ST;
            for (int j = issued; j < nB; ++j) {
                const int st = j % ST;
                if (j >= ST && !mbar_wait(kv_empty + st, ((j / ST) - 1) & 1, abort, W2_KV_EMPTY))
                    break;
                mbar_arrive_expect_tx(k_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sK + st * C::TILE + cb * C::BOX, &tmK, k_full + st, cb * 64,
                                kv_row0 + j * 128, (int)chain);
                mbar_arrive_expect_tx(v_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sV + st * C::TILE + cb * C::BOX, &tmV, v_full + st, cb * 64,
                                kv_row0 + j * 128, (int)chain);
                issued = j + 1;
            }
            if (*abort) {
                seg2_drain(q_full, 0);
                seg2_drain(m_full, 0);
                for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j) {
                    seg2_drain(k_full + j % ST, (j / ST) & 1);
                    seg2_drain(v_full + j % ST, (j / ST) & 1);
                }
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
            const uint32_t aQ[2] = {smem_u32(sQ[0]), smem_u32(sQ[1])};
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aM = smem_u32(sM);
            bool ok = mbar_wait(q_full, 0, abort, W2_Q);

            auto issue_s = [&](int x, int j) {
                const uint32_t kbase = aK + (j % ST) * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(T_S[x], sdesc_sw128(aQ[x] + off, 16, 1024),
                           sdesc_sw128(kbase + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + x);
            };
            auto issue_pv = [&](int x, int i) -> bool {
                if (!mbar_wait(p_full + x, i & 1, abort, W2_P)) return false;
                tc_fence_after();
                const uint32_t vbase = aV + (i % ST) * C::TILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = sdesc_sw128(vbase + kk * 2048, C::BOX, 1024);
                    mma_ts(T_O[x], T_S[x] + kk * 8, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
                }
                return true;
            };

            if (ok) ok = mbar_wait(k_full, 0, abort, W2_K);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            }
            for (int j = 1; ok && j < nB; ++j) {
                const int sp = (j - 1) % ST;
                if (!(ok = mbar_wait(v_full + sp, ((j - 1) / ST) & 1, abort, W2_V))) break;
                if (!(ok = issue_pv(0, j - 1))) break;
                if (!(ok = mbar_wait(k_full + j % ST, (j / ST) & 1, abort, W2_K))) break;
                tc_fence_after();
                if (j < nB - 1) issue_s(0, j);
                else mma_commit(pv_done + 0);          // tile A is complete
                if (!(ok = issue_pv(1, j - 1))) break;
                mma_commit(kv_empty + sp);
                issue_s(1, j);
            }
            if (ok) {
                const int last = nB - 1;
                ok = mbar_wait(v_full + last % ST, (last / ST) & 1, abort, W2_V);
                if (ok) ok = issue_pv(1, last);
                if (ok) {
                    mma_commit(pv_done + 1);
                    mma_commit(kv_empty + last % ST);
                }
            }
            if (ok) ok = mbar_wait(m_full, 0, abort, W2_M);
            for (int x = 0; ok && x < 2; ++x) {
                if (!(ok = mbar_wait(sq_full + x, 0, abort, W2_SQ))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(T_S[x], sdesc_sw128(aQ[x] + off, 16, 1024),
                           sdesc_sw128(aM + kk * 2048, C::MBOX, 1024), idO, kk > 0 ? 1u : 0u);
                }
                mma_commit(r_full + x);
            }
            mma_commit(mma_done);
            seg2_drain(mma_done, 0);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_HIGH));
        // ---------------------------------------------------------------- softmax / epilogue
        const int x = warp >> 2;                          // 0: tile A, 1: tile B
        const int r = threadIdx.x & 127;                  // query row within the tile
        const int qt = 2 * p + x;                         // q tile index inside the segment
        const int nX = nB - 1 + x;                        // key tiles this tile reads
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float *zsrc = a.snapZ + (chain * a.S + s) * (int64_t)D;
        for (int i = threadIdx.x; i < D; i += 256) sZ[i] = zsrc[i];
        asm volatile("bar.sync 1, 256;" ::: "memory");

        const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int i = 0; i < nX; ++i) {
            if (!(ok = mbar_wait(s_full + x, i & 1, abort, W2_S))) break;
            tc_fence_after();
            const bool diag = (i == qt);
            // the whole row of S in registers (one wait for four loads)
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + T_S[x] + c * 32, v[c]);
            tmem_ld_wait();
            if (diag) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (c * 32 + e > r) v[c][e] = __float_as_uint(-INFINITY);
            }
            // row maximum: three-input max, four independent partial maxima
            float pm[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) pm[u] = __uint_as_float(v[0][u]);
#pragma unroll
            for (int u = 4; u < 128; u += 2)
                pm[(u >> 1) & 3] = max3f(pm[(u >> 1) & 3], __uint_as_float(v[u >> 5][u & 31]),
                                         __uint_as_float(v[u >> 5][(u & 31) + 1]));
            const float mt = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
            const bool resc = (mt - m_used) * kscale > 8.f;
            float alpha = 1.f;
            if (resc) {
                alpha = ex2((m_used - mt) * kscale);
                m_used = mt;
                l *= alpha;
            }
            if (i > 0 && __any_sync(0xffffffffu, resc)) {
                // PV_X(i-1) is complete: the commit behind S_X(i) covers it
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + T_O[x] + c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(lane_base + T_O[x] + c, o);
                }
            }
            // P = exp2((S - m) * scale) in bf16, written over the S tile's first 64 columns
            const float mk = m_used * kscale;
            // scale-and-shift and the partial row sums on packed fp32 pairs
            const uint64_t ks2 = f2_pack(kscale, kscale), nm2 = f2_pack(-mk, -mk);
            uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float y0, y1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(v[c][2 * e]), __uint_as_float(v[c][2 * e + 1])),
                                     ks2, nm2), y0, y1);
                    const float p0 = ex2(y0), p1 = ex2(y1);
                    ps2[e & 3] = f2_add(ps2[e & 3], f2_pack(p0, p1));
                    pk[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16(lane_base + T_S[x] + c * 16, pk);
            }
            float rsum[8];
#pragma unroll
            for (int u = 0; u < 4; ++u) f2_unpack(ps2[u], rsum[2 * u], rsum[2 * u + 1]);
            const float rs = ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3])) + ((rsum[4] + rsum[5]) + (rsum[6] + rsum[7]));
            l += rs;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full + x);
        }
        if (ok) ok = mbar_wait(pv_done + x, 0, abort, W2_PV);
        if (ok) ok = mbar_wait(q_full, 0, abort, W2_Q);
        if (ok) {
            tc_fence_after();
            float dp[4] = {0.f, 0.f, 0.f, 0.f};       // sigma(q) . z in four partial sums
            uint8_t *q = sQ[x];
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 *ptr = reinterpret_cast<uint4 *>(q + cb * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4));
                    uint4 v = *ptr;
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                        float x0 = __low2float(t), x1 = __high2float(t);
                        x0 = elu1(x0);
                        x1 = elu1(x1);
                        const int c = cb * 64 + ch * 8 + 2 * e;
                        dp[e] = fmaf(x1, sZ[c + 1], fmaf(x0, sZ[c], dp[e]));
                        w[e] = pack_bf16x2(x0, x1);
                    }
                    *ptr = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(sq_full + x);
            const float den = (dp[0] + dp[1]) + (dp[2] + dp[3]);
            if (mbar_wait(r_full + x, 0, abort, W2_R)) {
                tc_fence_after();
                const float g = 1.f / (1.f + __expf(-a.beta[h]));
                const float wl = (1.f - g) / l;
                const float wm = den == 0.f ? 0.f : g / den;
                const int64_t row = (int64_t)s * a.N + (int64_t)qt * 128 + r;
                const bool live = row < a.L;                     // rows past L: not stored
                __nv_bfloat16 *orow = a.out + (bh * a.L + row) * D;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32], rr[32];
                    tmem_ld32(lane_base + T_O[x] + c, o);
                    tmem_ld32(lane_base + T_S[x] + c, rr);
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
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc
}  // namespace infini
