// Additive ("linear") memory chain on the 5th-generation tensor cores (sm_100a).
//
//   M_s = M_{s-1} + sigma(K_s)^T V_s,   z_s = z_{s-1} + sum_t sigma(k_t)
// (AI Wiki "Infini-Attention", "How does the compressive memory work?", the additive
// variant; the running sum of "What is linear attention and the delta rule?").
//
// One CTA per chain (b, kv head) keeps [M | z] for all d value columns in one fp32 TMEM
// accumulator (128 lanes = key features, columns 0..d-1 = M, column d = z) and walks the
// segments in order, 128 tokens at a time:
//   1. TMA brings K and V chunks (128-byte swizzle); the compute warpgroup turns the K tile
//      into sigma(K) in place (bf16).
//   2. One thread issues acc += sigma(K)^T [V | 1]: sigma(K) is the MN-major A operand, V the
//      MN-major B operand followed by a constant 64-column box whose first column is ones,
//      so one MMA chain (N = d + 16) accumulates both M and z.
//   3. At each segment end thread c reads row c of the accumulator and publishes the bf16
//      snapshot M_s[c, :] and z_s[c] that segment s + 1 reads, or M_out / z_out at the end.
// The accumulator starts from (M0, z0), so every snapshot is M0 + sum_{j<s} dM_j directly.
// d = 64 runs as d = 128 on the A side with a zero feature box.  All waits are bounded.
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

template <int D>
struct LinCfg {
    static constexpr int ST = 2;
    static constexpr int KBOX = 128 * 128;              // 128 rows x 64 bf16
    static constexpr int KTILE = 2 * KBOX;              // features padded to 128
    static constexpr int NVB = D / 64 + 1;              // V boxes + the constant ones box
    static constexpr int VTILE = NVB * KBOX;
    static constexpr int NACC = D + 16;                 // MMA N: M columns, z, padding
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + ST * KTILE;
    static constexpr int OFF_BAR = OFF_V + ST * VTILE;
    static constexpr int NBAR = 3 * ST + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 256;
};

struct LinArgs {
    const float *M0, *z0;      // may be NULL (zeros); may alias M_out / z_out exactly
    float *snapZ;              // [chains, S, D]
    __nv_bfloat16 *snapMb;     // [chains, S, D, D]
    float *M_out, *z_out;
    int N, S;
    int64_t L;                 // rows per chain: rows of the last segment past L count as absent
};

enum : int { WL_KV_EMPTY = 301, WL_A = 302, WL_KV_FULL = 303, WL_SEG = 304, WL_DRAIN = 305 };

__device__ __forceinline__ float sigma_lin(float x) { return elu1(x); }

template <int D>
__global__ void __launch_bounds__(256, 1)
k_linear_state_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const LinArgs a)
{
    static_assert(D == 64 || D == 128, "tensor-core linear chain: d = 64 or 128");
    using C = LinCfg<D>;
    constexpr int ST = C::ST;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int64_t chain = blockIdx.x;
    const int nch = a.N / 128;
    const int total = a.S * nch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + ST;
    // one a_ready per stage: the sigma pass may finish a chunk before the MMA thread has seen
    // the previous one, and a barrier waited by parity must not complete twice unobserved
    uint64_t *a_ready = bars + 2 * ST, *seg_done = a_ready + ST, *mma_done = seg_done + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(kv_full + i, 1);
            mbar_init(kv_empty + i, 1);
            mbar_init(a_ready + i, 128);
        }
        mbar_init(seg_done, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t T_ACC = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int issued = 0;
            for (int g = 0; g < total; ++g) {
                const int st = g % ST, s = g / nch, i = g % nch;
                if (g >= ST && !mbar_wait_short(kv_empty + st, ((g / ST) - 1) & 1, abort, WL_KV_EMPTY))
                    break;
                const int row = s * a.N + i * 128;
                mbar_arrive_expect_tx(kv_full + st, (uint32_t)(2 * D * 128 * 2));
                for (int kb = 0; kb < D / 64; ++kb) {
                    tma_load_3d(sK + st * C::KTILE + kb * C::KBOX, &tmK, kv_full + st, kb * 64, row,
                                (int)chain);
                    tma_load_3d(sV + st * C::VTILE + kb * C::KBOX, &tmV, kv_full + st, kb * 64, row,
                                (int)chain);
                }
                issued = g + 1;
            }
            if (*abort)
                for (int g = (issued > ST ? issued - ST : 0); g < issued; ++g) {
                    const long long t0 = clock64();
                    while (!mbar_try_wait(kv_full + g % ST, (g / ST) & 1))
                        if (clock64() - t0 > kSpinLimitCycles) {
                            atomicCAS(&g_wait_status, 0, WL_DRAIN);
                            break;
                        }
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idA = idesc_bf16(128, C::NACC, 1, 1);   // sigma(K)^T [V | 1]
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
            for (int g = 0; g < total; ++g) {
                const int st = g % ST, i = g % nch;
                if (!mbar_wait_short(a_ready + st, (g / ST) & 1, abort, WL_A)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {        // 128 tokens in steps of 16
                    const uint64_t ad = sdesc_sw128(aK + st * C::KTILE + kk * 2048, C::KBOX, 1024);
                    const uint64_t bd = sdesc_sw128(aV + st * C::VTILE + kk * 2048, C::KBOX, 1024);
                    mma_ss(T_ACC, ad, bd, idA, 1u);
                }
                mma_commit(kv_empty + st);
                if (i == nch - 1) mma_commit(seg_done);
            }
            mma_commit(mma_done);
            const long long t0 = clock64();
            while (!mbar_try_wait(mma_done, 0))
                if (clock64() - t0 > kSpinLimitCycles) {
                    atomicCAS(&g_wait_status, 0, WL_DRAIN);
                    break;
                }
        }
    } else if (warp >= 4) {
        const int r = threadIdx.x - 128;            // token row / key feature row
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        // constant box after V in every stage: column 0 = 1, the rest 0
        for (int i = r; i < ST * 128 * 8; i += 128) {
            const int st = i / (128 * 8), row = (i / 8) % 128, ch = i % 8;
            const uint32_t v = (ch == 0) ? 0x3F80u : 0u;   // bf16 1.0 in the lowest element
            *reinterpret_cast<uint4 *>(sV + st * C::VTILE + (D / 64) * C::KBOX + row * 128 +
                                       ((ch ^ (row & 7)) << 4)) = make_uint4(v, 0, 0, 0);
        }
        if (D == 64)
            for (int i = r; i < ST * C::KBOX / 16; i += 128) {
                const int st = i / (C::KBOX / 16), o = i % (C::KBOX / 16);
                reinterpret_cast<uint4 *>(sK + st * C::KTILE + C::KBOX)[o] = make_uint4(0, 0, 0, 0);
            }
        // accumulator row r <- [M0[r, :] | z0[r] | 0]
#pragma unroll 1
        for (int c0 = 0; c0 < C::NACC; c0 += 16) {
            uint32_t v16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int col = c0 + e;
                float x = 0.f;
                if (r < D) {
                    if (col < D) {
                        x = a.M0 ? a.M0[chain * D * D + (int64_t)r * D + col] : 0.f;
                        // slot 0 (what segment 0 reads) is the initial state itself
                        a.snapMb[chain * a.S * (int64_t)D * D + (int64_t)r * D + col] =
                            __float2bfloat16_rn(x);
                    } else if (col == D) {
                        x = a.z0 ? a.z0[chain * D + r] : 0.f;
                        a.snapZ[chain * a.S * (int64_t)D + r] = x;
                    }
                }
                v16[e] = __float_as_uint(x);
            }
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(lane_base + T_ACC + c0),
                "r"(v16[0]), "r"(v16[1]), "r"(v16[2]), "r"(v16[3]), "r"(v16[4]), "r"(v16[5]),
                "r"(v16[6]), "r"(v16[7]), "r"(v16[8]), "r"(v16[9]), "r"(v16[10]), "r"(v16[11]),
                "r"(v16[12]), "r"(v16[13]), "r"(v16[14]), "r"(v16[15])
                : "memory");
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        asm volatile("bar.sync 1, 128;" ::: "memory");

        for (int g = 0; g < total; ++g) {
            const int st = g % ST, s = g / nch, i = g % nch;
            if (!mbar_wait_short(kv_full + st, (g / ST) & 1, abort, WL_KV_FULL)) break;
            uint8_t *krow = sK + st * C::KTILE;
            // a row past L (the zero fill of a short last segment) gets sigma = 0, not sigma(0):
            // a mask, not a select, so the element loop stays free of branches
            const uint32_t keep = (int64_t)s * a.N + i * 128 + r < a.L ? 0xFFFFFFFFu : 0u;
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
                        w[e] = pack_bf16x2(sigma_lin(__low2float(t2)), sigma_lin(__high2float(t2))) & keep;
                    }
                    *p = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(a_ready + st);
            if (i == nch - 1) {
                if (!mbar_wait_short(seg_done, s & 1, abort, WL_SEG)) break;
                tc_fence_after();
                if (r < D) {
                    // row r of [M_s | z_s]
                    const bool last = (s + 1 == a.S);
                    const int64_t slot = chain * a.S + s + 1;
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(lane_base + T_ACC + c0, v);
                        tmem_ld_wait();
                        if (last) {
                            float4 *dst = reinterpret_cast<float4 *>(a.M_out + chain * D * D +
                                                                     (int64_t)r * D + c0);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                                     __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
                        } else {
                            uint32_t pk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                            uint4 *dst = reinterpret_cast<uint4 *>(a.snapMb + slot * D * D +
                                                                   (int64_t)r * D + c0);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                        }
                    }
                    uint32_t zv[32];
                    tmem_ld32(lane_base + T_ACC + D, zv);
                    tmem_ld_wait();
                    const float zc = __uint_as_float(zv[0]);
                    if (last) a.z_out[chain * D + r] = zc;
                    else a.snapZ[slot * D + r] = zc;
                } else {
                    // lanes past d still take part in the warp-wide loads
                    uint32_t v[32];
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        tmem_ld32(lane_base + T_ACC + c0, v);
                        tmem_ld_wait();
                    }
                    tmem_ld32(lane_base + T_ACC + D, v);
                    tmem_ld_wait();
                }
                tc_fence_before();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(T_ACC, C::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace infini
