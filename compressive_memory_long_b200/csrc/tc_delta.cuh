// Delta-rule memory chain on the 5th-generation tensor cores (sm_100a).
//
// For every (chain = (b, kv head)) and segment s, in order (AI Wiki "Infini-Attention",
// "How does the compressive memory work?"):
//   den_t = sigma(k_t) . z_{s-1}
//   U_t   = v_t - (den_t == 0 ? 0 : sigma(k_t) M_{s-1} / den_t)     (every token reads M_{s-1})
//   M_s   = M_{s-1} + sigma(K_s)^T U_s,      z_s = z_{s-1} + sum_t sigma(k_t)
// The update of value column e needs only column e of M_{s-1}, column e of V_s and the shared
// z, so each CTA owns CB = 16 value columns of one chain and walks all segments; the chain's
// d/16 CTAs run side by side.  sigma(K) is computed once per token beforehand
// (k_sigma_bf16) and read here through TMA.  Per 128-token chunk g:
//   1. TMA brings sigma(K) (128 x d, 128-byte swizzle) and V[:, cols] (128 x 16).
//   2. One thread issues R = sigma(K) B^T with B = [M^T | z | 0 | M_lo^T | z_lo | 0] (48 rows,
//      bf16: M and z split into hi + lo parts, side by side so one N = 48 MMA reads the
//      sigma(K) tile once; the lo half starts at row 24): R[0..15] + R[24..39] are the
//      prediction numerators, R[16] + R[40] is den_t.
//   3. Thread t forms U_t and writes [U_hi | 1 | 0 | U_lo | 0]^T (the residual is a small
//      difference of large terms: one bf16 rounding of it would cost ~1e-2 of M).
//   4. One thread issues Macc += sigma(K)^T [U_hi | 1 | 0 | U_lo | 0] (sigma(K) read as the
//      MN-major operand): M[:, cols] = Macc[0..15] + Macc[24..39], z = Macc[16], in fp32.
// Within a segment every R reads the same M_{s-1}, so R(g+1) is issued before the update of
// chunk g (R accumulators and U tiles double-buffered); only the first chunk of a segment
// waits for B (the initial state, or the boundary where thread c -- TMEM lane c = key
// feature c -- reads its row of Macc,
// publishes the bf16 snapshot M_s[c, cols] (and z_s from the chain's first CTA) for the
// segment kernel, and rewrites the B operand).  d = 64 runs as d = 128 with zero features.
// All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

// sigma(x) = ELU(x) + 1 of every element, bf16 in and out, 8 elements per thread and step.
__global__ void __launch_bounds__(256)
k_sigma_bf16(const __nv_bfloat16 *__restrict__ x, __nv_bfloat16 *__restrict__ y, int64_t n8)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(x);
    uint4 *dst = reinterpret_cast<uint4 *>(y);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = src[i];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
            float a = __low2float(t), b = __high2float(t);
            a = elu1(a);
            b = elu1(b);
            w[e] = pack_bf16x2(a, b);
        }
        dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

struct ChainCfg {
    static constexpr int CB = 16;                 // value columns per CTA
    static constexpr int NB = 48;                 // rows of the B operands (hi half, lo half)
    static constexpr int LO = 24;                 // first row of the lo half (a multiple of 8)
    static constexpr int ST = 4;                  // sigma(K)/V stages
    static constexpr int KBOX = 128 * 128;        // 128 rows x 64 bf16
    static constexpr int KTILE = 2 * KBOX;        // 128 tokens x 128 features (padded)
    static constexpr int VTILE = 128 * CB * 2;    // 128 tokens x 16 bf16, unswizzled
    static constexpr int BBOX = NB * 128;         // 48 rows x 64 bf16
    static constexpr int BTILE = 2 * BBOX;        // 48 rows x 128 (features or tokens)
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + ST * KTILE;
    static constexpr int OFF_B = OFF_V + ST * VTILE;    // [M | z]^T, hi and lo halves
    static constexpr int OFF_U = OFF_B + BTILE;         // 2 x [U | 1]^T, hi and lo halves
    static constexpr int OFF_BAR = OFF_U + 2 * BTILE;
    static constexpr int NBAR = 2 * ST + 8;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(OFF_B % 1024 == 0 && OFF_U % 1024 == 0, "operand tiles must be 1024-aligned");
};

struct ChainArgs {
    const float *snapM;        // slot 0 (fp32) of every chain: M0
    const float *snapZ_in;     // slot 0 of every chain: z0
    float *snapZ;              // [chains, S, D]: z_{s-1} for s >= 1 written here
    __nv_bfloat16 *snapMb;     // [chains, S, D, D]: bf16 M_{s-1} for s >= 1 written here
    float *M_out, *z_out;
    int N, S;
};

enum : int { WC_KV_EMPTY = 201, WC_B = 202, WC_U = 203, WC_KV_FULL = 204, WC_R = 205,
             WC_UPD = 206, WC_DRAIN = 207 };

__device__ __forceinline__ void chain_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kSpinLimitCycles) {
            atomicCAS(&g_wait_status, 0, WC_DRAIN);
            return;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(256, 1)
k_delta_chain_tc(const __grid_constant__ CUtensorMap tmSK, const __grid_constant__ CUtensorMap tmV,
                 const ChainArgs a)
{
    static_assert(D == 64 || D == 128, "tensor-core delta chain: d = 64 or 128");
    using C = ChainCfg;
    constexpr int ST = C::ST, CB = C::CB;
    constexpr int NBLK = D / CB;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int64_t chain = blockIdx.x / NBLK;
    const int cb = (blockIdx.x % NBLK) * CB;
    const int nch = a.N / 128;
    const int total = a.S * nch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sB = smem + C::OFF_B;
    uint8_t *sU = smem + C::OFF_U;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + ST;
    uint64_t *r_full = bars + 2 * ST, *u_ready = r_full + 2, *upd_done = u_ready + 2;
    uint64_t *b_ready = upd_done + 2, *mma_done = b_ready + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(kv_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(r_full + i, 1);
            mbar_init(u_ready + i, 128);
            mbar_init(upd_done + i, 1);
        }
        mbar_init(b_ready, 128);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_M = tmem;
    const uint32_t T_R[2] = {tmem + 64, tmem + 128};

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmSK);
            prefetch_tmap(&tmV);
            int issued = 0;
            for (int g = 0; g < total; ++g) {
                const int st = g % ST, s = g / nch, i = g % nch;
                if (g >= ST && !mbar_wait_short(kv_empty + st, ((g / ST) - 1) & 1, abort, WC_KV_EMPTY))
                    break;
                const int row = s * a.N + i * 128;
                mbar_arrive_expect_tx(kv_full + st, (uint32_t)(D * 128 * 2 + C::VTILE));
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_3d(sK + st * C::KTILE + kb * C::KBOX, &tmSK, kv_full + st, kb * 64, row,
                                (int)chain);
                tma_load_3d(sV + st * C::VTILE, &tmV, kv_full + st, cb, row, (int)chain);
                issued = g + 1;
            }
            if (*abort)
                for (int g = (issued > ST ? issued - ST : 0); g < issued; ++g)
                    chain_drain(kv_full + g % ST, (g / ST) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idR = idesc_bf16(128, C::NB, 0, 0);   // sigma(K) . B^T
            constexpr uint32_t idU = idesc_bf16(128, C::NB, 1, 0);   // sigma(K)^T . [U | 1]
            const uint32_t aK = smem_u32(sK), aB = smem_u32(sB), aU = smem_u32(sU);
            auto issue_r = [&](int g) -> bool {
                // the first chunk of segment s waits for B holding M_{s-1}: phase 0 is the
                // initial state written in the prologue, phase s the boundary after segment s-1
                if (g % nch == 0 && !mbar_wait_short(b_ready, (g / nch) & 1, abort, WC_B))
                    return false;
                if (!mbar_wait_short(kv_full + g % ST, (g / ST) & 1, abort, WC_KV_FULL)) return false;
                tc_fence_after();
                const uint32_t kbase = aK + (g % ST) * C::KTILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {        // K = 128 features in steps of 16
                    const uint32_t off = (kk >> 2) * C::KBOX + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_R[g & 1], sdesc_sw128(kbase + off, 16, 1024),
                           sdesc_sw128(aB + boff, 16, 1024), idR, kk > 0 ? 1u : 0u);
                }
                mma_commit(r_full + (g & 1));
                return true;
            };
            auto issue_update = [&](int g) -> bool {
                const int bb = g & 1;
                if (!mbar_wait_short(u_ready + bb, (g >> 1) & 1, abort, WC_U)) return false;
                tc_fence_after();
                const uint32_t kbase = aK + (g % ST) * C::KTILE;
                const uint32_t ub = aU + bb * C::BTILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {        // K = 128 tokens in steps of 16
                    const uint64_t ad = sdesc_sw128(kbase + kk * 2048, C::KBOX, 1024);
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_M, ad, sdesc_sw128(ub + boff, 16, 1024), idU, 1u);
                }
                mma_commit(kv_empty + g % ST);
                mma_commit(upd_done + bb);
                return true;
            };
            bool ok = issue_r(0);
            for (int g = 0; ok && g < total; ++g) {
                const bool next_starts_segment = (g + 1) % nch == 0;
                if (g + 1 < total && !next_starts_segment) ok = issue_r(g + 1);
                if (ok) ok = issue_update(g);
                if (ok && g + 1 < total && next_starts_segment) ok = issue_r(g + 1);
            }
            mma_commit(mma_done);
            chain_drain(mma_done, 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- compute warpgroup
        const int r = threadIdx.x - 128;           // token row of a chunk / key feature row
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
        // constant rows of both [U | 1]^T tiles: 16 = ones, 17..23 and 40..47 = zeros
        for (int i = r; i < 2 * 2 * 16 * 64; i += 128) {
            const int buf = i / (2 * 16 * 64), box = (i / (16 * 64)) % 2, k16 = (i / 64) % 16;
            const int rr = k16 < 8 ? 16 + k16 : 32 + k16;           // 16..23, 40..47
            const int t = i % 64;
            *reinterpret_cast<__nv_bfloat16 *>(sU + buf * C::BTILE + box * C::BBOX + rr * 128 +
                                               ((((t >> 3) ^ (rr & 7))) << 4) + (t & 7) * 2) =
                rr == 16 ? one : zero;
        }
        if (D == 64)   // the padded feature box of every stage stays zero
            for (int i = r; i < ST * C::KBOX / 16; i += 128) {
                const int st = i / (C::KBOX / 16), o = i % (C::KBOX / 16);
                reinterpret_cast<uint4 *>(sK + st * C::KTILE + C::KBOX)[o] = make_uint4(0, 0, 0, 0);
            }
        // column c of B: rows 0..15 = M[c, cols] hi, 16 = z[c] hi, 32..47 / 48 = lo parts
        auto write_b_col = [&](int c, const float *m16, float zc) {
            const int box = c >> 6, cc = c & 63;
#pragma unroll 1
            for (int e = 0; e < C::LO; ++e) {
                const float x = e < CB ? m16[e] : (e == CB ? zc : 0.f);
                const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                const int o = box * C::BBOX + ((((cc >> 3) ^ (e & 7))) << 4) + (cc & 7) * 2;
                *reinterpret_cast<__nv_bfloat16 *>(sB + o + e * 128) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(sB + o + (C::LO + e) * 128) = lo;
            }
        };
        {
            float m16[CB];
            float zc = 0.f;
#pragma unroll
            for (int e = 0; e < CB; ++e) m16[e] = 0.f;
            if (r < D) {
                const float *src = a.snapM + chain * a.S * (int64_t)D * D + (int64_t)r * D + cb;
#pragma unroll
                for (int e = 0; e < CB; ++e) m16[e] = src[e];
                zc = a.snapZ_in[chain * a.S * (int64_t)D + r];
            }
            uint32_t acc[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
                acc[e] = __float_as_uint(e < CB ? m16[e] : (e == CB ? zc : 0.f));
            tmem_st32(lane_base + T_M, acc);
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0u;
            tmem_st32(lane_base + T_M + 32, acc);
            tmem_st_wait();
            write_b_col(r, m16, zc);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_ready);                       // B holds the initial state

        bool ok = true;
        for (int g = 0; ok && g < total; ++g) {
            const int st = g % ST, s = g / nch, i = g % nch, bb = g & 1;
            if (!(ok = mbar_wait_short(kv_full + st, (g / ST) & 1, abort, WC_KV_FULL))) break;
            // this token's 16 values of V in chunk g
            float vv[CB];
            {
                const uint4 *vp = reinterpret_cast<const uint4 *>(sV + st * C::VTILE + r * CB * 2);
                uint4 v0 = vp[0], v1 = vp[1];
                uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    __nv_bfloat162 t2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                    vv[2 * e] = __low2float(t2);
                    vv[2 * e + 1] = __high2float(t2);
                }
            }
            if (!(ok = mbar_wait_short(r_full + bb, (g >> 1) & 1, abort, WC_R))) break;
            tc_fence_after();
            uint32_t rh[32], rl[32];
            tmem_ld32(lane_base + T_R[bb], rh);
            tmem_ld32(lane_base + T_R[bb] + C::LO, rl);
            tmem_ld_wait();
            const float den = __uint_as_float(rh[CB]) + __uint_as_float(rl[CB]);
            const float inv = den == 0.f ? 0.f : 1.f / den;
            // U tile bb is free once the update of chunk g-2 has completed
            if (g >= 2 && !(ok = mbar_wait_short(upd_done + bb, ((g >> 1) - 1) & 1, abort, WC_UPD))) break;
            {
                const int box = r >> 6, tt = r & 63;
                uint8_t *ub = sU + bb * C::BTILE + box * C::BBOX + (tt & 7) * 2;
#pragma unroll
                for (int e = 0; e < CB; ++e) {
                    const float u = vv[e] - (__uint_as_float(rh[e]) + __uint_as_float(rl[e])) * inv;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(u);
                    const int o = ((((tt >> 3) ^ (e & 7))) << 4);
                    *reinterpret_cast<__nv_bfloat16 *>(ub + o + e * 128) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(ub + o + (C::LO + e) * 128) =
                        __float2bfloat16_rn(u - __bfloat162float(hi));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(u_ready + bb);

            if (i == nch - 1) {
                // segment end: M_s, z_s from the accumulator (lane r = key feature r)
                if (!(ok = mbar_wait_short(upd_done + bb, (g >> 1) & 1, abort, WC_UPD))) break;
                tc_fence_after();
                uint32_t acc[32], acl[32];
                tmem_ld32(lane_base + T_M, acc);
                tmem_ld32(lane_base + T_M + C::LO, acl);
                tmem_ld_wait();
                float m16[CB];
#pragma unroll
                for (int e = 0; e < CB; ++e) m16[e] = __uint_as_float(acc[e]) + __uint_as_float(acl[e]);
                const float zc = __uint_as_float(acc[CB]);
                if (r < D) {
                    if (s + 1 < a.S) {
                        const int64_t slot = chain * a.S + s + 1;
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(m16[2 * e], m16[2 * e + 1]);
                        uint4 *dst = reinterpret_cast<uint4 *>(a.snapMb + slot * D * D + (int64_t)r * D + cb);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        if (cb == 0) a.snapZ[slot * D + r] = zc;
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(a.M_out + chain * D * D + (int64_t)r * D + cb);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_float4(m16[4 * e], m16[4 * e + 1], m16[4 * e + 2], m16[4 * e + 3]);
                        if (cb == 0) a.z_out[chain * D + r] = zc;
                    }
                }
                if (g + 1 < total) {
                    write_b_col(r, m16, zc);
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(b_ready);           // R of the next segment may read M_s
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace tc
}  // namespace infini
