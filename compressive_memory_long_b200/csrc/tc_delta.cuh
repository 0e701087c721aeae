// Delta-rule memory chain on the 5th-generation tensor cores (sm_100a).
//
// For every (chain = (b, kv head)) and segment s, in order (AI Wiki "Infini-Attention",
// "How does the compressive memory work?"):
//   den_t = sigma(k_t) . z_{s-1}
//   U_t   = v_t - (den_t == 0 ? 0 : sigma(k_t) M_{s-1} / den_t)     (every token reads M_{s-1})
//   M_s   = M_{s-1} + sigma(K_s)^T U_s,      z_s = z_{s-1} + sum_t sigma(k_t)
// The update of value column e needs only column e of M_{s-1}, column e of V_s and the shared
// z, so each CTA owns CB = 16 value columns of one chain and walks all segments; the chain's
// D/16 CTAs run side by side.  Per 128-token chunk:
//   1. TMA brings K (128 x d, 128-byte swizzle) and V[:, cols] (128 x 16) into a stage.
//   2. The compute warpgroup (thread t = token t) overwrites its K row with sigma(K) in bf16.
//   3. One thread issues R = sigma(K) [M_{s-1}^T | z_{s-1}]^T with M and z split into bf16
//      hi + lo parts (two accumulating MMAs, N = 32): columns 0..15 are the prediction
//      numerators, column 16 is den_t.
//   4. Thread t forms U_t and writes U^T split into bf16 hi + lo parts (the residual is a
//      small difference of large terms, so one bf16 rounding of it would cost ~1e-2 of M),
//      next to a constant row of ones (hi part) / zeros (lo part).
//   5. One thread issues Macc += sigma(K)^T [U_hi | 1] + sigma(K)^T [U_lo | 0] (sigma(K) read
//      as the MN-major operand): columns 0..15 of the TMEM accumulator carry M[:, cols] in
//      fp32, column 16 carries z.
// At each segment end thread c (TMEM lane c = key feature c) reads its row of Macc, publishes
// the bf16 snapshot M_s[c, cols] (and z_s from the chain's first CTA) for the segment kernel,
// and refreshes the hi/lo operand copies.  d = 64 runs as d = 128 with zero columns.
// All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

struct ChainCfg {
    static constexpr int CB = 16;                 // value columns per CTA
    static constexpr int NB = 32;                 // rows of the B operands: 16 + z/ones + pad
    static constexpr int ST = 2;                  // K/V stages
    static constexpr int KBOX = 128 * 128;        // 128 rows x 64 bf16
    static constexpr int KTILE = 2 * KBOX;        // 128 tokens x 128 features (padded)
    static constexpr int VTILE = 128 * CB * 2;    // 128 tokens x 16 bf16, unswizzled
    static constexpr int BBOX = NB * 128;         // 32 rows x 64 bf16
    static constexpr int BTILE = 2 * BBOX;        // 32 rows x 128 (features or tokens)
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + ST * KTILE;
    static constexpr int OFF_BH = OFF_V + ST * VTILE;   // [M | z]^T hi   (32 x 128 features)
    static constexpr int OFF_BL = OFF_BH + BTILE;       // [M | z]^T lo
    static constexpr int OFF_U = OFF_BL + BTILE;        // [U_hi | 1]^T   (32 x 128 tokens)
    static constexpr int OFF_UL = OFF_U + BTILE;        // [U_lo | 0]^T
    static constexpr int OFF_BAR = OFF_UL + BTILE;
    static constexpr int NBAR = 2 * ST + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(OFF_BH % 1024 == 0 && OFF_U % 1024 == 0 && OFF_UL % 1024 == 0,
                  "operand tiles must be 1024-aligned");
};

struct ChainArgs {
    const float *snapM;        // slot 0 (fp32) of every chain: M0
    const float *snapZ_in;     // slot 0 of every chain: z0
    float *snapZ;              // [chains, S, D]: z_{s-1} for s >= 1 written here
    __nv_bfloat16 *snapMb;     // [chains, S, D, D]: bf16 M_{s-1} for s >= 1 written here
    float *M_out, *z_out;
    int N, S;
};

enum : int { WC_KV_EMPTY = 201, WC_A = 202, WC_U = 203, WC_KV_FULL = 204, WC_R = 205,
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

__device__ __forceinline__ float sigma_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }

template <int D>
__global__ void __launch_bounds__(256, 1)
k_delta_chain_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
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
    uint8_t *sBH = smem + C::OFF_BH;
    uint8_t *sBL = smem + C::OFF_BL;
    uint8_t *sU = smem + C::OFF_U;
    uint8_t *sUL = smem + C::OFF_UL;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + ST;
    uint64_t *a_ready = bars + 2 * ST, *r_full = a_ready + 1, *u_ready = r_full + 1;
    uint64_t *upd_done = u_ready + 1, *mma_done = upd_done + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(kv_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        mbar_init(a_ready, 128);
        mbar_init(r_full, 1);
        mbar_init(u_ready, 128);
        mbar_init(upd_done, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_M = tmem, T_R = tmem + 32;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int issued = 0;
            for (int g = 0; g < total; ++g) {
                const int st = g % ST, s = g / nch, i = g % nch;
                if (g >= ST && !mbar_wait(kv_empty + st, ((g / ST) - 1) & 1, abort, WC_KV_EMPTY))
                    break;
                const int row = s * a.N + i * 128;
                mbar_arrive_expect_tx(kv_full + st, (uint32_t)(D * 128 * 2 + C::VTILE));
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_3d(sK + st * C::KTILE + kb * C::KBOX, &tmK, kv_full + st, kb * 64, row,
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
            constexpr uint32_t idU = idesc_bf16(128, C::NB, 1, 0);   // sigma(K)^T . [U|1]
            const uint32_t aK = smem_u32(sK), aBH = smem_u32(sBH), aBL = smem_u32(sBL);
            const uint32_t aU = smem_u32(sU), aUL = smem_u32(sUL);
            for (int g = 0; g < total; ++g) {
                const int st = g % ST;
                if (!mbar_wait(a_ready, g & 1, abort, WC_A)) break;
                tc_fence_after();
                const uint32_t kbase = aK + st * C::KTILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {        // K = 128 features in steps of 16
                    const uint32_t off = (kk >> 2) * C::KBOX + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_R, sdesc_sw128(kbase + off, 16, 1024), sdesc_sw128(aBH + boff, 16, 1024),
                           idR, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * C::KBOX + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_R, sdesc_sw128(kbase + off, 16, 1024), sdesc_sw128(aBL + boff, 16, 1024),
                           idR, 1u);
                }
                mma_commit(r_full);
                if (!mbar_wait(u_ready, g & 1, abort, WC_U)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {        // K = 128 tokens in steps of 16
                    const uint64_t ad = sdesc_sw128(kbase + kk * 2048, C::KBOX, 1024);
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_M, ad, sdesc_sw128(aU + boff, 16, 1024), idU, 1u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sdesc_sw128(kbase + kk * 2048, C::KBOX, 1024);
                    const uint32_t boff = (kk >> 2) * C::BBOX + (kk & 3) * 32;
                    mma_ss(T_M, ad, sdesc_sw128(aUL + boff, 16, 1024), idU, 1u);
                }
                mma_commit(kv_empty + st);
                mma_commit(upd_done);
            }
            mma_commit(mma_done);
            chain_drain(mma_done, 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- compute warpgroup
        const int r = threadIdx.x - 128;           // token row of a chunk / key feature row
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
        // constant rows: [U_hi | 1]^T row 16 = ones, rows 17..31 = zeros; [U_lo | 0]^T rows
        // 16..31 = zeros (both token boxes)
        for (int i = r; i < 2 * 16 * 64; i += 128) {
            const int box = i / (16 * 64), rr = 16 + (i / 64) % 16, t = i % 64;
            const int o = box * C::BBOX + rr * 128 + ((((t >> 3) ^ (rr & 7))) << 4) + (t & 7) * 2;
            *reinterpret_cast<__nv_bfloat16 *>(sU + o) = rr == 16 ? one : zero;
            *reinterpret_cast<__nv_bfloat16 *>(sUL + o) = zero;
        }
        if (D == 64)   // the padded feature box of every K stage stays zero
            for (int i = r; i < ST * C::KBOX / 16; i += 128) {
                const int st = i / (C::KBOX / 16), o = i % (C::KBOX / 16);
                reinterpret_cast<uint4 *>(sK + st * C::KTILE + C::KBOX)[o] = make_uint4(0, 0, 0, 0);
            }
        // initial state: lane/row c = r holds [M0[c, cols] | z0[c] | 0 ...]
        auto write_b_col = [&](int c, const float *m16, float zc) {
            // column c of the 32 x 128 hi / lo operands, rows 0..15 = M, 16 = z, 17.. = 0
            const int box = c >> 6, cc = c & 63;
            for (int e = 0; e < C::NB; ++e) {
                const float x = e < CB ? m16[e] : (e == CB ? zc : 0.f);
                const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                const int o = box * C::BBOX + e * 128 + ((((cc >> 3) ^ (e & 7))) << 4) + (cc & 7) * 2;
                *reinterpret_cast<__nv_bfloat16 *>(sBH + o) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(sBL + o) = lo;
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
            tmem_st_wait();
            write_b_col(r, m16, zc);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        asm volatile("bar.sync 1, 128;" ::: "memory");

        bool ok = true;
        for (int g = 0; ok && g < total; ++g) {
            const int st = g % ST, s = g / nch, i = g % nch;
            if (!(ok = mbar_wait(kv_full + st, (g / ST) & 1, abort, WC_KV_FULL))) break;
            // sigma(K) in place, row r
            uint8_t *krow = sK + st * C::KTILE;
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 *p = reinterpret_cast<uint4 *>(krow + kb * C::KBOX + r * 128 +
                                                         ((ch ^ (r & 7)) << 4));
                    uint4 v = *p;
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 t2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                        w[e] = pack_bf16x2(sigma_f(__low2float(t2)), sigma_f(__high2float(t2)));
                    }
                    *p = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(a_ready);
            // this token's 16 values of V
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
            if (!(ok = mbar_wait(r_full, g & 1, abort, WC_R))) break;
            tc_fence_after();
            uint32_t rr[32];
            tmem_ld32(lane_base + T_R, rr);
            tmem_ld_wait();
            const float den = __uint_as_float(rr[CB]);
            const float inv = den == 0.f ? 0.f : 1.f / den;
            // sU is free once the previous chunk's update has completed
            if (g > 0 && !(ok = mbar_wait(upd_done, (g - 1) & 1, abort, WC_UPD))) break;
            {
                const int box = r >> 6, tt = r & 63;
#pragma unroll
                for (int e = 0; e < CB; ++e) {
                    const float u = vv[e] - __uint_as_float(rr[e]) * inv;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(u);
                    const int o = box * C::BBOX + e * 128 + ((((tt >> 3) ^ (e & 7))) << 4) + (tt & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16 *>(sU + o) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sUL + o) =
                        __float2bfloat16_rn(u - __bfloat162float(hi));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(u_ready);

            if (i == nch - 1) {
                // segment end: M_s, z_s from the accumulator (lane r = key feature r)
                if (!(ok = mbar_wait(upd_done, g & 1, abort, WC_UPD))) break;
                tc_fence_after();
                uint32_t acc[32];
                tmem_ld32(lane_base + T_M, acc);
                tmem_ld_wait();
                float m16[CB];
#pragma unroll
                for (int e = 0; e < CB; ++e) m16[e] = __uint_as_float(acc[e]);
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
                write_b_col(r, m16, zc);
                fence_proxy_async_smem();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

}  // namespace tc
}  // namespace infini
