// Local-attention part of the backward pass on the tensor cores (sm_100a, bf16, d = 64 or
// 128, N % 128 == 0; with 64-token segments the row statistics, dq and dk / dv take a pair
// of segments as one 128-row tile: N = 128 and ceil(S / 2) segments in their arguments,
// `pair` set, a block-diagonal causal mask, and the row statistics' two halves retrieve
// from their own segments' memories; G^M and the update keep one CTA per segment and read
// a 64-token segment as the first half of the 128-row tile they load, the other half being
// rows past the segment's end, which they zero).
//
// Same arithmetic as k_bwd_dq / k_bwd_dkdv (backward.cuh; AI Wiki "Infini-Attention", "What
// happens inside the Infini-attention block?", the local causal softmax of each segment):
// with lse and D_i = dA_dot_i . A_dot_i from k_bwd_rows, g = sigmoid(beta_h),
//   P = exp2(S log2(e) / sqrt(d) - lse),  dS = P * ((1 - g) dout V^T - D),
//   dq += dS K / sqrt(d),  dk += dS^T Q / sqrt(d),  dv += (1 - g) P^T dout,
// over the causal keys of the row's own segment.  P and dS enter the second products as
// bf16 (the operands of kind::f16), every product accumulates in fp32 in TMEM.
//
//   k_bwd_dq_tc    one CTA per (b, h, segment, 128 query rows); per key tile:
//                  S = Q K^T and dP = dout V^T into TMEM, dS (bf16) over S, dQ += dS K
//   k_bwd_dkdv_tc  one CTA per (b, kv head, segment, 128 keys), over the group's query
//                  heads and the query tiles at or after the key tile; per query tile:
//                  S^T = K Q^T and dP^T = V dout^T, (1 - g) P^T over S^T and dS^T over
//                  dP^T (bf16), dV += P^T dout, dK += dS^T Q; each key row has one owner
//   k_bwd_rows_tc  one CTA per (b, h, segment, 128 query rows): the forward of the rows
//                  (S = Q K^T, online softmax, O += P V; sigma(Q) over Q, R = sigma(Q) M and
//                  dout M^T from one bf16 M tile read MN-major and K-major), then per row
//                  lse, D = (1 - g) dout . A_dot, the retrieval factors g / den and dden, the
//                  retrieval part of dq and the gate's partial sum
//   k_bwd_gm_tc    one CTA per (b, kv head, segment): G^M_s = sum over the group's rows of
//                  (wsc sigma(q))^T dout and G^z_s = sum sigma(q) dden in one product
//                  [wsc sigma(Q)]^T [dout | dden / wsc] (the extra column is 0 where wsc is:
//                  dden is 0 there too); wsc sigma(Q) is written over the staged Q tile
//   k_bwd_update_tc one CTA per (b, kv head, segment), per 128-token tile: dU = sigma(K) dM_s
//                  (dv += dU) and, for the delta rule, sigma(K) M_{s-1} = den R; then
//                  dsigma(k) = U dM_s^T - (dU / den) M_{s-1}^T + dden z with U = v - R,
//                  dden = dU . R / den, and h_s += sigma(K)^T dden; linear: dsigma(k) = V dM_s^T.
//                  dM_s and M_{s-1} enter as bf16 hi + lo tiles (read MN-major and K-major):
//                  one rounding of them is shared by every row, so its error would add up
//                  coherently in h_s; dden enters as hi + lo columns
// Roles: warps 0-3 one thread per row (elementwise work, epilogue); warp 4 loads (TMA; in
// k_bwd_dkdv_tc its 32 lanes also stage the query tile's lse and D); warp 5 lane 0 issues
// the MMAs.  All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"
#include "tc_segment_p.cuh"

namespace infini {
namespace tc {

template <int D>
struct BwdTcCfg {
    static_assert(D == 64 || D == 128, "tensor-core backward: d = 64 or 128");
    static constexpr int THREADS = 192;
    static constexpr int TILE = 128 * D * 2;          // 128 rows x d bf16
    static constexpr int BOX = 128 * 128;             // 128 rows x 64 bf16
    static constexpr int ST = 2;                      // stages of the streamed operands
    // dq: Q | dout | ST x (K | V);  dkdv: K | V | ST x (Q | dout | lse | D)
    static constexpr int OFF_A = 0, OFF_B = TILE, OFF_RING = 2 * TILE;
    static constexpr int RING_DQ = 2 * TILE;
    static constexpr int RING_KV = 2 * TILE + 2 * 128 * 4;
    static constexpr int OFF_BAR_DQ = OFF_RING + ST * RING_DQ;
    static constexpr int OFF_BAR_KV = OFF_RING + ST * RING_KV;
    static constexpr int NBAR = 3 * ST + 6;
    static constexpr int ALLOC_DQ = OFF_BAR_DQ + NBAR * 8 + 16 + 1024;
    static constexpr int ALLOC_KV = OFF_BAR_KV + NBAR * 8 + 16 + 1024;
    static_assert(ALLOC_DQ <= 227 * 1024 && ALLOC_KV <= 227 * 1024, "shared memory");
    // TMEM: S (or S^T) [0,128), dP (or dP^T) [128,256), then the accumulators
    static constexpr uint32_t T_S = 0, T_P = 128, T_A0 = 256, T_A1 = 256 + D;
};

struct BwdTcArgs {
    const float *beta;
    const float *lse, *Drow;      // [B, H, L] from k_bwd_rows
    const float *dq_mem;          // [B, H, L, D]: the retrieval part of dq
    __nv_bfloat16 *dq;            // [B, H, L, D] output
    float *dk, *dv;               // [B, Hkv, L, D]: the local parts (fp32)
    int64_t L;
    int N, S, H, Hkv;
    int pair;                     // 1: a tile is two 64-token segments (N = 128 here)
};

// Outputs of the row statistics (the same buffers as k_bwd_rows writes)
struct BwdRowsArgs {
    const float *beta;
    const float *snapZ;           // [chains * S, D]: z_{s-1}
    float *lse, *Drow, *wsc, *dden;   // [B, H, L]
    float *dq_mem;                // [B, H, L, D]
    float *dbeta_part;            // [B, H, S, qparts]: qparts 64-row parts per segment
    int64_t L;
    int N, S, H, Hkv, qparts;
    int pair;                     // 1: a tile is two 64-token segments (N = 128, S = pairs here)
    int Sr;                       // the real segment count (snapshots, z, dbeta parts) when pair
};

template <int D>
struct BwdRowsCfg {
    static constexpr int TILE = 128 * D * 2, BOX = 128 * 128, ST = 2;
    static constexpr int MBYTES = D * D * 2, MBOX = D * 128;
    static constexpr int OFF_Q = 0, OFF_O = TILE, OFF_RING = 2 * TILE;      // ring: ST x (K | V)
    static constexpr int OFF_M = OFF_RING + ST * 2 * TILE;
    static constexpr int OFF_Z = OFF_M + MBYTES;      // z of the segment (of both, for a pair)
    static constexpr int OFF_RED = OFF_Z + 2 * D * 4; // 4 warp partial sums of the gate term
    static constexpr int NBAR = 3 * ST + 10;
    static constexpr int OFF_BAR = OFF_RED + 16;
    static constexpr int ALLOC = OFF_BAR + NBAR * 8 + 16 + 1024;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    // TMEM: S [0,128), O, R = sigma(Q) M, dout M^T (d columns each).  At d = 64 dout M^T
    // takes S's first columns (free once the last P V has run: MMAs execute in issue order),
    // so the kernel fits 256 columns and two CTAs share an SM.
    static constexpr uint32_t T_S = 0, T_O = 128, T_R = 128 + D, T_DM = D == 64 ? 0 : 128 + 2 * D;
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256 : 512;
};

struct BwdGmArgs {
    const float *wsc, *dden;      // [B, H, L] from the row statistics
    float *GM, *Gz;               // [chains * S, D, D], [chains * S, D]
    int64_t L;
    int N, S, H, Hkv;
};

template <int D>
struct BwdGmCfg {
    // one stage at d = 64: the stage's 64 KB then lets three CTAs share an SM (most d = 64
    // workloads have one or few steps per CTA); two at d = 128, whose CTAs walk the group's
    // heads over long segments
    static constexpr int BOX = 128 * 128, NB = D / 64, ST = D == 64 ? 1 : 2;
    // stage: A = wsc sigma(Q) over Q (features padded to 128 with a zero box at d = 64) |
    //        dout (NB boxes) | the extra column's box
    static constexpr int OFF_AQ = 0, OFF_DO = 2 * BOX, OFF_EX = OFF_DO + NB * BOX;
    static constexpr int STAGE = OFF_EX + BOX;
    static constexpr int NBAR = 3 * ST + 1;
    static constexpr int OFF_BAR = ST * STAGE;
    static constexpr int ALLOC = OFF_BAR + NBAR * 8 + 16 + 1024;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    static constexpr int NACC = D + 16;                    // G^M columns, then the G^z column
    static constexpr uint32_t TMEM_COLS = NACC <= 128 ? 128 : 256;
};

struct BwdUpdArgs {
    const float *dMs, *snapM, *snapZ;   // [chains * S, D, D], [chains * S, D, D], [chains * S, D]
    float *dv, *dsk, *h;                // [B, Hkv, L, D] (+=), [B, Hkv, L, D], [chains * S, D]
    int64_t L;
    int N, S;
};

template <int D>
struct BwdUpdCfg {
    static constexpr int BOX = 128 * 128, NB = D / 64, MBOX = D * 128, MBYTES = D * D * 2;
    // sigma(K) over K (features padded to 128 with a zero box at d = 64), then -dU / den over it
    // | V, then U | the dden columns' box | dM_s hi, lo | M_{s-1} hi, lo (bf16) | z
    static constexpr int OFF_K = 0, OFF_V = 2 * BOX, OFF_E = OFF_V + NB * BOX;
    static constexpr int OFF_DM = OFF_E + BOX, OFF_M = OFF_DM + 2 * MBYTES, OFF_Z = OFF_M + 2 * MBYTES;
    static constexpr int NBAR = 9;
    static constexpr int OFF_BAR = OFF_Z + D * 4;
    static constexpr int ALLOC = OFF_BAR + NBAR * 8 + 16 + 1024;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    // TMEM: dU | sigma(K) M | dsigma(k) (d columns each) | h (16); at d = 64 that fits 256
    // columns, so two CTAs share an SM (shared memory allows it too)
    static constexpr uint32_t T_1 = 0, T_2 = D, T_3 = 2 * D, T_H = 3 * D;
    static constexpr uint32_t TMEM_COLS = 3 * D + 16 <= 256 ? 256 : 512;
};

enum : int { WB_QF = 901, WB_KF = 902, WB_VF = 903, WB_KVE = 904, WB_SDP = 905, WB_DS = 906,
             WB_DONE = 907, WB_FULL = 908, WB_EMPTY = 909, WB_DRAIN = 910, WB_MF = 911,
             WB_SQ = 912, WB_RF = 913, WB_RED = 914, WB_UR = 915, WB_P3 = 916, WB_RH = 917 };

__device__ __forceinline__ void bwdtc_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WB_DRAIN);
            return;
        }
    }
}

// dq of 128 query rows: the retrieval part (from k_bwd_rows) plus dS K / sqrt(d)
template <int D>
__global__ void __launch_bounds__(192, 1)
k_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
            const BwdTcArgs a)
{
    using C = BwdTcCfg<D>;
    constexpr int ST = C::ST;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int qtiles = a.N / 128;
    int64_t bid = blockIdx.x;
    const int qt = qtiles - 1 - (int)(bid % qtiles);          // the longest rows first
    bid /= qtiles;
    const int s = (int)(bid % a.S);
    const int64_t bh = bid / a.S;
    const int h = (int)(bh % a.H);
    const int64_t chain = (bh / a.H) * a.Hkv + h / (a.H / a.Hkv);
    const int64_t seg0 = (int64_t)s * a.N;
    const int valid = (int)(a.L - seg0 < a.N ? a.L - seg0 : a.N);
    const int q0 = qt * 128;
    if (q0 >= valid) return;
    const int nk = qt + 1;                                      // key tiles 0..qt
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sQ = smem + C::OFF_A, *sO = smem + C::OFF_B;
    auto sK = [&](int st) { return smem + C::OFF_RING + st * C::RING_DQ; };
    auto sV = [&](int st) { return smem + C::OFF_RING + st * C::RING_DQ + C::TILE; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR_DQ);
    uint64_t *k_full = bars, *v_full = bars + ST, *kv_empty = bars + 2 * ST;
    uint64_t *q_full = bars + 3 * ST, *sdp_full = q_full + 1, *ds_full = q_full + 2, *dq_done = q_full + 3;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR_DQ + C::NBAR * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_BAR_DQ + C::NBAR * 8 + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        mbar_init(q_full, 1);
        mbar_init(sdp_full, 1);
        mbar_init(ds_full, 128);
        mbar_init(dq_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------------------------- loads
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmO);
            mbar_arrive_expect_tx(q_full, 2 * C::TILE);
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_3d(sQ + cb * C::BOX, &tmQ, q_full, cb * 64, (int)(seg0 + q0), (int)bh);
                tma_load_3d(sO + cb * C::BOX, &tmO, q_full, cb * 64, (int)(seg0 + q0), (int)bh);
            }
            int issued = 0;
            for (int j = 0; j < nk; ++j) {
                const int st = j % ST;
                if (j >= ST && !mbar_wait_short(kv_empty + st, ((j / ST) - 1) & 1, abort, WB_KVE)) break;
                mbar_arrive_expect_tx(k_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sK(st) + cb * C::BOX, &tmK, k_full + st, cb * 64, (int)(seg0 + j * 128),
                                (int)chain);
                mbar_arrive_expect_tx(v_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sV(st) + cb * C::BOX, &tmV, v_full + st, cb * 64, (int)(seg0 + j * 128),
                                (int)chain);
                issued = j + 1;
            }
            if (*abort) {
                bwdtc_drain(q_full, 0);
                for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j) {
                    bwdtc_drain(k_full + j % ST, (j / ST) & 1);
                    bwdtc_drain(v_full + j % ST, (j / ST) & 1);
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
            const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO);
            bool ok = mbar_wait_short(q_full, 0, abort, WB_QF);
            for (int j = 0; ok && j < nk; ++j) {
                const int st = j % ST;
                const uint32_t aK = smem_u32(sK(st)), aV = smem_u32(sV(st));
                if (!(ok = mbar_wait_short(k_full + st, (j / ST) & 1, abort, WB_KF))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {        // S = Q K^T
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + C::T_S, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                if (!(ok = mbar_wait_short(v_full + st, (j / ST) & 1, abort, WB_VF))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {        // dP = dout V^T
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + C::T_P, sdesc_sw128(aO + off, 16, 1024), sdesc_sw128(aV + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(sdp_full);
                if (!(ok = mbar_wait_short(ds_full, j & 1, abort, WB_DS))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)                 // dQ += dS K (dS in S's columns)
                    mma_ts(tmem + C::T_A0, tmem + C::T_S + kk * 8, sdesc_sw128(aK + kk * 2048, C::BOX, 1024),
                           idO, (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(kv_empty + st);
            }
            mma_commit(dq_done);
            bwdtc_drain(dq_done, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- rows
        const int r = threadIdx.x;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int64_t row = bh * a.L + seg0 + q0 + r;
        const bool live = q0 + r < valid;
        const float lse = live ? a.lse[row] : 0.f, Dr = live ? a.Drow[row] : 0.f;
        const float c1 = 1.f - 1.f / (1.f + __expf(-a.beta[h]));
        const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
        const int lo = a.pair && r >= 64 ? 64 : 0;             // a pair's second segment: its own keys
        bool ok = true;
        for (int j = 0; ok && j < nk; ++j) {
            if (!(ok = mbar_wait(sdp_full, j & 1, abort, WB_SDP))) break;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[2][32], pv[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    tmem_ld32(lane_base + tmem + C::T_S + half * 64 + c * 32, sv[c]);
                    tmem_ld32(lane_base + tmem + C::T_P + half * 64 + c * 32, pv[c]);
                }
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float ds2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int col = half * 64 + c * 32 + 2 * e + u;       // key in the tile
                            const bool vis = live && j * 128 + col < valid && (j < qt || col <= r) && col >= lo;
                            const float p = vis ? ex2(fmaf(__uint_as_float(sv[c][2 * e + u]), sl2, -lse)) : 0.f;
                            ds2[u] = p * fmaf(c1, __uint_as_float(pv[c][2 * e + u]), -Dr);
                        }
                        pk[e] = pack_bf16x2(ds2[0], ds2[1]);
                    }
                    tmem_st16(lane_base + tmem + C::T_S + half * 32 + c * 16, pk);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        if (ok && mbar_wait(dq_done, 0, abort, WB_DONE)) {
            tc_fence_after();
            const float rs = rsqrtf((float)D);
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t o[32];
                tmem_ld32(lane_base + tmem + C::T_A0 + c, o);
                tmem_ld_wait();
                if (live) {
                    const float4 *src = reinterpret_cast<const float4 *>(a.dq_mem + row * D + c);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 m = src[e];
                        pk[2 * e] = pack_bf16x2(fmaf(__uint_as_float(o[4 * e]), rs, m.x),
                                                fmaf(__uint_as_float(o[4 * e + 1]), rs, m.y));
                        pk[2 * e + 1] = pack_bf16x2(fmaf(__uint_as_float(o[4 * e + 2]), rs, m.z),
                                                    fmaf(__uint_as_float(o[4 * e + 3]), rs, m.w));
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(a.dq + row * D + c);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// local dk, dv of 128 keys over the group's query heads and the query tiles at or after
// the key tile
template <int D>
__global__ void __launch_bounds__(192, 1)
k_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const BwdTcArgs a)
{
    using C = BwdTcCfg<D>;
    constexpr int ST = C::ST;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int ktiles = a.N / 128;
    int64_t bid = blockIdx.x;
    const int kt = (int)(bid % ktiles);                      // the longest key tiles first
    bid /= ktiles;
    const int s = (int)(bid % a.S);
    const int64_t chain = bid / a.S;                         // b * Hkv + kv head
    const int G = a.H / a.Hkv;
    const int64_t bh0 = (chain / a.Hkv) * a.H + (chain % a.Hkv) * G;   // first query head
    const int64_t seg0 = (int64_t)s * a.N;
    const int valid = (int)(a.L - seg0 < a.N ? a.L - seg0 : a.N);
    const int k0 = kt * 128;
    if (k0 >= valid) return;
    const int nq = (valid - k0 + 127) / 128;                 // query tiles kt .. kt + nq - 1
    const int steps = G * nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sK = smem + C::OFF_A, *sV = smem + C::OFF_B;
    auto sQ = [&](int st) { return smem + C::OFF_RING + st * C::RING_KV; };
    auto sO = [&](int st) { return smem + C::OFF_RING + st * C::RING_KV + C::TILE; };
    auto sL = [&](int st) { return reinterpret_cast<float *>(smem + C::OFF_RING + st * C::RING_KV + 2 * C::TILE); };
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR_KV);
    uint64_t *full = bars, *empty = bars + ST, *kv_full = bars + 3 * ST;
    uint64_t *sdp_full = kv_full + 1, *ps_full = kv_full + 2, *done = kv_full + 3;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR_KV + C::NBAR * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_BAR_KV + C::NBAR * 8 + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(full + i, 33);          // the TMA lane's expect_tx + the 32 lanes' lse / D
            mbar_init(empty + i, 1);
        }
        mbar_init(kv_full, 1);
        mbar_init(sdp_full, 1);
        mbar_init(ps_full, 128);
        mbar_init(done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        // -------------------------------------------------------------------- loads
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmO);
            mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_3d(sK + cb * C::BOX, &tmK, kv_full, cb * 64, (int)(seg0 + k0), (int)chain);
                tma_load_3d(sV + cb * C::BOX, &tmV, kv_full, cb * 64, (int)(seg0 + k0), (int)chain);
            }
        }
        int issued = 0;
        bool ok = true;
        for (int i = 0; i < steps; ++i) {
            const int st = i % ST;
            const int64_t bh = bh0 + i / nq;
            const int q0 = k0 + (i % nq) * 128;
            if (i >= ST && !(ok = mbar_wait_short(empty + st, ((i / ST) - 1) & 1, abort, WB_EMPTY))) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(full + st, 2 * C::TILE);
                for (int cb = 0; cb < D / 64; ++cb) {
                    tma_load_3d(sQ(st) + cb * C::BOX, &tmQ, full + st, cb * 64, (int)(seg0 + q0), (int)bh);
                    tma_load_3d(sO(st) + cb * C::BOX, &tmO, full + st, cb * 64, (int)(seg0 + q0), (int)bh);
                }
            }
            // lse and D of the tile's 128 query rows (0 past the segment's valid rows)
            float *sl = sL(st);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int jr = lane * 4 + u;
                const bool in = q0 + jr < valid;
                const int64_t row = bh * a.L + seg0 + q0 + jr;
                sl[jr] = in ? a.lse[row] : 0.f;
                sl[128 + jr] = in ? a.Drow[row] : 0.f;
            }
            mbar_arrive(full + st);
            issued = i + 1;
        }
        if (lane == 0 && (*abort || !ok)) {
            bwdtc_drain(kv_full, 0);
            for (int i = (issued > ST ? issued - ST : 0); i < issued; ++i) bwdtc_drain(full + i % ST, (i / ST) & 1);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait_short(kv_full, 0, abort, WB_KF);
            for (int i = 0; ok && i < steps; ++i) {
                const int st = i % ST;
                const uint32_t aQ = smem_u32(sQ(st)), aO = smem_u32(sO(st));
                if (!(ok = mbar_wait_short(full + st, (i / ST) & 1, abort, WB_FULL))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {        // S^T = K Q^T, dP^T = V dout^T
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + C::T_S, sdesc_sw128(aK + off, 16, 1024), sdesc_sw128(aQ + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::T_P, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(aO + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(sdp_full);
                if (!(ok = mbar_wait_short(ps_full, i & 1, abort, WB_DS))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {               // dV += P^T dout, dK += dS^T Q
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    mma_ts(tmem + C::T_A0, tmem + C::T_S + kk * 8, sdesc_sw128(aO + kk * 2048, C::BOX, 1024),
                           idO, acc);
                    mma_ts(tmem + C::T_A1, tmem + C::T_P + kk * 8, sdesc_sw128(aQ + kk * 2048, C::BOX, 1024),
                           idO, acc);
                }
                mma_commit(empty + st);
            }
            mma_commit(done);
            bwdtc_drain(done, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- key rows
        const int r = threadIdx.x;                               // key row of the tile
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const bool live = k0 + r < valid;
        const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
        const int hi = a.pair && r < 64 ? 64 : 128;            // a pair's first segment: its own queries
        bool ok = true;
        for (int i = 0; ok && i < steps; ++i) {
            const int st = i % ST;
            const int h = (int)((bh0 + i / nq) % a.H);
            const int qrel = (i % nq) * 128;                     // query tile - key tile, in rows
            const float c1 = 1.f - 1.f / (1.f + __expf(-a.beta[h]));
            // the producer's lse / D writes are visible after this wait
            if (!(ok = mbar_wait(full + st, (i / ST) & 1, abort, WB_FULL))) break;
            if (!(ok = mbar_wait(sdp_full, i & 1, abort, WB_SDP))) break;
            tc_fence_after();
            const float *sl = sL(st);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[2][32], pv[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    tmem_ld32(lane_base + tmem + C::T_S + half * 64 + c * 32, sv[c]);
                    tmem_ld32(lane_base + tmem + C::T_P + half * 64 + c * 32, pv[c]);
                }
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pp[16], dd[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float p2[2], d2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int col = half * 64 + c * 32 + 2 * e + u;   // query in the tile
                            // causal: query row >= key row; rows past the segment's end out
                            const bool vis = live && (qrel > 0 || col >= r) && k0 + qrel + col < valid && col < hi;
                            const float p = vis ? ex2(fmaf(__uint_as_float(sv[c][2 * e + u]), sl2, -sl[col])) : 0.f;
                            p2[u] = c1 * p;
                            d2[u] = p * fmaf(c1, __uint_as_float(pv[c][2 * e + u]), -sl[128 + col]);
                        }
                        pp[e] = pack_bf16x2(p2[0], p2[1]);
                        dd[e] = pack_bf16x2(d2[0], d2[1]);
                    }
                    tmem_st16(lane_base + tmem + C::T_S + half * 32 + c * 16, pp);
                    tmem_st16(lane_base + tmem + C::T_P + half * 32 + c * 16, dd);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ps_full);
        }
        if (ok && mbar_wait(done, 0, abort, WB_DONE)) {
            tc_fence_after();
            const float rs = rsqrtf((float)D);
            const int64_t krow = chain * a.L + seg0 + k0 + r;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t v32[32], k32[32];
                tmem_ld32(lane_base + tmem + C::T_A0 + c, v32);
                tmem_ld32(lane_base + tmem + C::T_A1 + c, k32);
                tmem_ld_wait();
                if (live) {
                    float4 *dv = reinterpret_cast<float4 *>(a.dv + krow * D + c);
                    float4 *dk = reinterpret_cast<float4 *>(a.dk + krow * D + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        dv[e] = make_float4(__uint_as_float(v32[4 * e]), __uint_as_float(v32[4 * e + 1]),
                                            __uint_as_float(v32[4 * e + 2]), __uint_as_float(v32[4 * e + 3]));
                        dk[e] = make_float4(__uint_as_float(k32[4 * e]) * rs, __uint_as_float(k32[4 * e + 1]) * rs,
                                            __uint_as_float(k32[4 * e + 2]) * rs, __uint_as_float(k32[4 * e + 3]) * rs);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}


// the forward of 128 query rows and the backward's row statistics (at d = 64 two CTAs per
// SM: 256 TMEM columns, ~108 KB of shared memory, at most 168 registers)
template <int D>
__global__ void __launch_bounds__(192, D == 64 ? 2 : 1)
k_bwd_rows_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const __grid_constant__ CUtensorMap tmM, const BwdRowsArgs a)
{
    using C = BwdRowsCfg<D>;
    constexpr int ST = C::ST;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int qtiles = a.N / 128;
    int64_t bid = blockIdx.x;
    const int qt = qtiles - 1 - (int)(bid % qtiles);          // the longest rows first
    bid /= qtiles;
    const int s = (int)(bid % a.S);
    const int64_t bh = bid / a.S;
    const int h = (int)(bh % a.H);
    const int64_t chain = (bh / a.H) * a.Hkv + h / (a.H / a.Hkv);
    const int64_t seg0 = (int64_t)s * a.N;
    const int valid = (int)(a.L - seg0 < a.N ? a.L - seg0 : a.N);
    const int q0 = qt * 128;
    // a pair: rows 0-63 are segment 2s and read its memory, rows 64-127 segment 2s + 1 (when
    // it exists); the gate's parts are laid out per real segment
    const int Ssnap = a.pair ? a.Sr : a.S;
    const int sA = a.pair ? 2 * s : s;
    const bool hasB = a.pair && sA + 1 < a.Sr;
    float *part = a.pair ? a.dbeta_part + bh * a.Sr + sA
                         : a.dbeta_part + (bh * a.S + s) * a.qparts + 2 * qt;   // two 64-row parts
    const int nparts = a.pair && !hasB ? 1 : 2;
    if (q0 >= valid) {
        if (threadIdx.x < nparts) part[threadIdx.x] = 0.f;
        return;
    }
    const int nk = qt + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sQ = smem + C::OFF_Q, *sO = smem + C::OFF_O, *sM = smem + C::OFF_M;
    float *sZ = reinterpret_cast<float *>(smem + C::OFF_Z);
    float *sRed = reinterpret_cast<float *>(smem + C::OFF_RED);
    auto sK = [&](int st) { return smem + C::OFF_RING + st * 2 * C::TILE; };
    auto sV = [&](int st) { return smem + C::OFF_RING + st * 2 * C::TILE + C::TILE; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *k_full = bars, *v_full = bars + ST, *kv_empty = bars + 2 * ST;
    uint64_t *q_full = bars + 3 * ST, *m_full = q_full + 1, *s_full = q_full + 2, *p_full = q_full + 3;
    uint64_t *sq_full = q_full + 4, *r_full = q_full + 5, *red_full = q_full + 6, *mma_done = q_full + 7;
    // a pair's second half: its R and dout M^T (r_full2), once the first half's rows have
    // read theirs from the same TMEM columns (r_half)
    uint64_t *r_full2 = q_full + 8, *r_half = q_full + 9;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + C::NBAR * 8 + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        mbar_init(q_full, 1);
        mbar_init(m_full, 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(sq_full, 128);
        mbar_init(r_full, 1);
        mbar_init(red_full, 4);
        mbar_init(mma_done, 1);
        mbar_init(r_full2, 1);
        mbar_init(r_half, 64);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(tmem_holder, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------------------------- loads
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmO);
            prefetch_tmap(&tmM);
            mbar_arrive_expect_tx(q_full, 2 * C::TILE);
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_3d(sQ + cb * C::BOX, &tmQ, q_full, cb * 64, (int)(seg0 + q0), (int)bh);
                tma_load_3d(sO + cb * C::BOX, &tmO, q_full, cb * 64, (int)(seg0 + q0), (int)bh);
            }
            // M_{s-1} (and for a pair's second segment its own memory, in the key ring's second
            // slot, which the single key tile of a pair leaves free) with z
            const int nm = hasB ? 2 : 1;
            mbar_arrive_expect_tx(m_full, nm * (C::MBYTES + D * 4));
            for (int x = 0; x < nm; ++x)
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d((x ? sK(1) : sM) + cb * C::MBOX, &tmM, m_full, cb * 64, 0,
                                (int)(chain * Ssnap + sA + x));
            bulk_load(sZ, a.snapZ + (chain * Ssnap + sA) * (int64_t)D, nm * D * 4, m_full);
            int issued = 0;
            for (int j = 0; j < nk; ++j) {
                const int st = j % ST;
                if (j >= ST && !mbar_wait_short(kv_empty + st, ((j / ST) - 1) & 1, abort, WB_KVE)) break;
                mbar_arrive_expect_tx(k_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sK(st) + cb * C::BOX, &tmK, k_full + st, cb * 64, (int)(seg0 + j * 128),
                                (int)chain);
                mbar_arrive_expect_tx(v_full + st, C::TILE);
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(sV(st) + cb * C::BOX, &tmV, v_full + st, cb * 64, (int)(seg0 + j * 128),
                                (int)chain);
                issued = j + 1;
            }
            if (*abort) {
                bwdtc_drain(q_full, 0);
                bwdtc_drain(m_full, 0);
                for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j) {
                    bwdtc_drain(k_full + j % ST, (j / ST) & 1);
                    bwdtc_drain(v_full + j % ST, (j / ST) & 1);
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);     // B MN-major (V; M for R)
            constexpr uint32_t idK = idesc_bf16(128, D, 0, 0);     // B K-major (M for dout M^T)
            const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO), aM = smem_u32(sM);
            bool ok = mbar_wait_short(q_full, 0, abort, WB_QF);
            for (int j = 0; ok && j < nk; ++j) {
                const int st = j % ST;
                const uint32_t aK = smem_u32(sK(st)), aV = smem_u32(sV(st));
                if (!(ok = mbar_wait_short(k_full + st, (j / ST) & 1, abort, WB_KF))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {        // S = Q K^T
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + C::T_S, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
                if (!(ok = mbar_wait_short(p_full, j & 1, abort, WB_DS))) break;
                if (!(ok = mbar_wait_short(v_full + st, (j / ST) & 1, abort, WB_VF))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)                 // O += P V (P in S's columns)
                    mma_ts(tmem + C::T_O, tmem + C::T_S + kk * 8, sdesc_sw128(aV + kk * 2048, C::BOX, 1024),
                           idO, (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(kv_empty + st);
            }
            if (ok) ok = mbar_wait_short(m_full, 0, abort, WB_MF);
            if (ok) ok = mbar_wait_short(sq_full, 0, abort, WB_SQ);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    // R = sigma(Q) M: B = M, rows a (key features) along K, MN-major
                    mma_ss(tmem + C::T_R, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aM + kk * 2048, C::MBOX, 1024),
                           idO, kk > 0 ? 1u : 0u);
                    // dout M^T: B[c][a] = M[a][c], value columns c along K: K-major
                    mma_ss(tmem + C::T_DM, sdesc_sw128(aO + off, 16, 1024),
                           sdesc_sw128(aM + (kk >> 2) * C::MBOX + (kk & 3) * 32, 16, 1024), idK, kk > 0 ? 1u : 0u);
                }
                mma_commit(r_full);
            }
            if (ok && hasB) ok = mbar_wait_short(r_half, 0, abort, WB_RH);
            if (ok && hasB) {
                tc_fence_after();
                const uint32_t aM2 = smem_u32(sK(1));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + C::T_R, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aM2 + kk * 2048, C::MBOX, 1024),
                           idO, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::T_DM, sdesc_sw128(aO + off, 16, 1024),
                           sdesc_sw128(aM2 + (kk >> 2) * C::MBOX + (kk & 3) * 32, 16, 1024), idK, kk > 0 ? 1u : 0u);
                }
                mma_commit(r_full2);
            }
            mma_commit(mma_done);
            bwdtc_drain(mma_done, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- rows
        const int r = threadIdx.x;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const bool live = q0 + r < valid;
        const bool second = a.pair && r >= 64;                  // a pair's second segment
        const float *zr = sZ + (second ? D : 0);
        const int lo = second ? 64 : 0;                          // the first key this row may see
        const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
        const float g = 1.f / (1.f + __expf(-a.beta[h]));
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; ok && j < nk; ++j) {
            if (!(ok = mbar_wait(s_full, j & 1, abort, WB_SDP))) break;
            tc_fence_after();
            const bool diag = (j == qt);
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + tmem + C::T_S + c * 32, v[c]);
            tmem_ld_wait();
            if (diag) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (c * 32 + e > r || c * 32 + e < lo) v[c][e] = __float_as_uint(-INFINITY);
            }
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
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                // PV(j-1) is complete: the commit behind S(j) covers it
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + tmem + C::T_O + c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(lane_base + tmem + C::T_O + c, o);
                }
            }
            const float mk = m_used * kscale;
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
                tmem_st16(lane_base + tmem + C::T_S + c * 16, pk);
            }
            float rsum[8];
#pragma unroll
            for (int u = 0; u < 4; ++u) f2_unpack(ps2[u], rsum[2 * u], rsum[2 * u + 1]);
            l += ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3])) + ((rsum[4] + rsum[5]) + (rsum[6] + rsum[7]));
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // sigma(Q) over this row (every Q K^T has completed) and den = sigma(q) . z
        float den = 0.f;
        if (ok) ok = mbar_wait(q_full, 0, abort, WB_QF);
        if (ok) ok = mbar_wait(m_full, 0, abort, WB_MF);
        if (ok) {
            den = segp_sigma_row<0, D, D / 8>(sQ, r, zr);
            fence_proxy_async_smem();
            mbar_arrive(sq_full);
        }
        float gm = 0.f;
        if (ok && (ok = mbar_wait(second && hasB ? r_full2 : r_full, 0, abort, WB_RF))) {
            tc_fence_after();
            // per row: A_dot = O / l, A_mem = R / den; dd = dout . A_dot, dam = dout . A_mem
            const float inv_l = 1.f / l;
            const float inv_den = den == 0.f ? 0.f : 1.f / den;
            float dd = 0.f, dam = 0.f;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t o[32], rr[32];
                tmem_ld32(lane_base + tmem + C::T_O + c, o);
                tmem_ld32(lane_base + tmem + C::T_R + c, rr);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int ch = ((c & 63) >> 3) + e;
                    const uint4 x = *reinterpret_cast<const uint4 *>(sO + (c >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4));
                    const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float d0 = __uint_as_float(w4[u] << 16), d1 = __uint_as_float(w4[u] & 0xffff0000u);
                        const int i0 = 8 * e + 2 * u;
                        dd = fmaf(d0, __uint_as_float(o[i0]) * inv_l, fmaf(d1, __uint_as_float(o[i0 + 1]) * inv_l, dd));
                        dam = fmaf(d0, __uint_as_float(rr[i0]) * inv_den, fmaf(d1, __uint_as_float(rr[i0 + 1]) * inv_den, dam));
                    }
                }
            }
            const float wsc = den == 0.f ? 0.f : g * inv_den;
            const float ddn = den == 0.f ? 0.f : -g * dam * inv_den;
            gm = live ? dam - dd : 0.f;
            const int64_t row = bh * a.L + seg0 + q0 + r;
            if (live) {
                a.lse[row] = m_used * kscale + __log2f(l);
                a.Drow[row] = (1.f - g) * dd;
                a.wsc[row] = wsc;
                a.dden[row] = ddn;
            }
            // the retrieval part of dq: (wsc dout M^T + dden z) * sigma'(q), sigma' = min(sigma, 1)
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t dm[32];
                tmem_ld32(lane_base + tmem + C::T_DM + c, dm);
                tmem_ld_wait();
                if (live) {
                    float4 *dst = reinterpret_cast<float4 *>(a.dq_mem + row * D + c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ch = ((c & 63) >> 3) + e;
                        const uint4 x = *reinterpret_cast<const uint4 *>(sQ + (c >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4));
                        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
                        float y[8];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float s0 = __uint_as_float(w4[u] << 16), s1 = __uint_as_float(w4[u] & 0xffff0000u);
                            const int i0 = 8 * e + 2 * u;
                            y[2 * u] = fmaf(wsc, __uint_as_float(dm[i0]), ddn * zr[c + i0]) * fminf(s0, 1.f);
                            y[2 * u + 1] = fmaf(wsc, __uint_as_float(dm[i0 + 1]), ddn * zr[c + i0 + 1]) * fminf(s1, 1.f);
                        }
                        dst[2 * e] = make_float4(y[0], y[1], y[2], y[3]);
                        dst[2 * e + 1] = make_float4(y[4], y[5], y[6], y[7]);
                    }
                }
            }
            if (hasB && !second) {
                // this row's R and dout M^T have been read: the second half's may replace them
                tc_fence_before();
                mbar_arrive(r_half);
            }
        }
        // the gate's partial sums: rows 0-63 and 64-127 of the tile, each in a fixed order
        if (ok) {
            float t = gm;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == 0) {
                sRed[warp] = t;
                mbar_arrive(red_full);
            }
            if (threadIdx.x == 0 && mbar_wait(red_full, 0, abort, WB_RED)) {
                part[0] = g * (1.f - g) * (sRed[0] + sRed[1]);
                if (nparts > 1) part[1] = g * (1.f - g) * (sRed[2] + sRed[3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}


// G^M_s and G^z_s of one (b, kv head, segment)
template <int D>
__global__ void __launch_bounds__(192, 1)
k_bwd_gm_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
            const BwdGmArgs a)
{
    using C = BwdGmCfg<D>;
    constexpr int ST = C::ST;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int64_t cs = blockIdx.x;                           // chain * S + s
    const int64_t chain = cs / a.S;
    const int s = (int)(cs % a.S);
    const int G = a.H / a.Hkv;
    const int64_t bh0 = (chain / a.Hkv) * a.H + (chain % a.Hkv) * G;
    const int64_t seg0 = (int64_t)s * a.N;
    const int valid = (int)(a.L - seg0 < a.N ? a.L - seg0 : a.N);
    const int nt = (valid + 127) / 128;                      // 128-row tiles of the segment
    const int steps = G * nt;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto stage = [&](int st) { return smem + st * C::STAGE; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars, *ready = bars + ST, *empty = bars + 2 * ST, *done = bars + 3 * ST;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + C::NBAR * 8 + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(full + i, 1);
            mbar_init(ready + i, 128);
            mbar_init(empty + i, 1);
        }
        mbar_init(done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (D == 64)       // the padded feature box of both stages' A tiles stays zero
        for (int i = threadIdx.x; i < ST * (C::BOX / 16); i += blockDim.x)
            reinterpret_cast<uint4 *>(stage(i / (C::BOX / 16)) + C::OFF_AQ + C::BOX)[i % (C::BOX / 16)] =
                make_uint4(0, 0, 0, 0);
    if (warp == 5) tmem_alloc(tmem_holder, C::TMEM_COLS);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------------------------- loads
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmO);
            int issued = 0;
            for (int i = 0; i < steps; ++i) {
                const int st = i % ST;
                const int64_t bh = bh0 + i / nt;
                const int row = (int)(seg0 + (i % nt) * 128);
                if (i >= ST && !mbar_wait_short(empty + st, ((i / ST) - 1) & 1, abort, WB_EMPTY)) break;
                mbar_arrive_expect_tx(full + st, 2 * C::NB * C::BOX);
                for (int cb = 0; cb < C::NB; ++cb) {
                    tma_load_3d(stage(st) + C::OFF_AQ + cb * C::BOX, &tmQ, full + st, cb * 64, row, (int)bh);
                    tma_load_3d(stage(st) + C::OFF_DO + cb * C::BOX, &tmO, full + st, cb * 64, row, (int)bh);
                }
                issued = i + 1;
            }
            if (*abort)
                for (int i = (issued > ST ? issued - ST : 0); i < issued; ++i)
                    bwdtc_drain(full + i % ST, (i / ST) & 1);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t id = idesc_bf16(128, C::NACC, 1, 1);    // both operands MN-major
            bool ok = true;
            for (int i = 0; ok && i < steps; ++i) {
                const int st = i % ST;
                if (!(ok = mbar_wait_short(ready + st, (i / ST) & 1, abort, WB_DS))) break;
                tc_fence_after();
                const uint32_t aA = smem_u32(stage(st) + C::OFF_AQ), aB = smem_u32(stage(st) + C::OFF_DO);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)                 // 16 rows per step
                    mma_ss(tmem, sdesc_sw128(aA + kk * 2048, C::BOX, 1024), sdesc_sw128(aB + kk * 2048, C::BOX, 1024),
                           id, (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty + st);
            }
            mma_commit(done);
            bwdtc_drain(done, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- rows
        const int r = threadIdx.x;
        bool ok = true;
        for (int i = 0; ok && i < steps; ++i) {
            const int st = i % ST;
            const int64_t bh = bh0 + i / nt;
            const int t = (i % nt) * 128 + r;                    // row in the segment
            const bool in = t < valid;
            const float wsc = in ? a.wsc[bh * a.L + seg0 + t] : 0.f;
            const float dd = in ? a.dden[bh * a.L + seg0 + t] : 0.f;
            if (!(ok = mbar_wait(full + st, (i / ST) & 1, abort, WB_FULL))) break;
            // A row = wsc sigma(q) over the Q row, in place (the TMA wrote it; the wait above
            // makes it visible); the extra column dden / wsc
            uint8_t *q = stage(st) + C::OFF_AQ;
            const uint64_t one2 = f2_pack(1.f, 1.f);
            const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
            const uint64_t w2 = f2_pack(wsc, wsc);
#pragma unroll 4
            for (int c0 = 0; c0 < D; c0 += 8) {
                const int ch = (c0 & 63) >> 3;
                uint4 *ptr = reinterpret_cast<uint4 *>(q + (c0 >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4));
                const uint4 x = *ptr;
                uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = __uint_as_float(w4[e] << 16), x1 = __uint_as_float(w4[e] & 0xffff0000u);
                    float a0, a1, p0, p1;
                    f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
                    f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
                    float y0, y1;
                    f2_unpack(f2_mul(f2_pack(fmaxf(p0, ex2(a0)), fmaxf(p1, ex2(a1))), w2), y0, y1);
                    w4[e] = pack_bf16x2(y0, y1);
                }
                *ptr = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            uint8_t *ex = stage(st) + C::OFF_EX + r * 128;
            const uint32_t e0 = pack_bf16x2(wsc == 0.f ? 0.f : dd / wsc, 0.f);
            *reinterpret_cast<uint4 *>(ex + ((0 ^ (r & 7)) << 4)) = make_uint4(e0, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(ex + ((1 ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();
            mbar_arrive(ready + st);
        }
        // lane a of the accumulator is key feature a: row a of G^M and G^z[a]
        if (ok && mbar_wait(done, 0, abort, WB_DONE)) {
            tc_fence_after();
            const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
            const bool live = r < D;
#pragma unroll 1
            for (int c = 0; c < C::NACC; c += 16) {
                uint32_t x[16];
                tmem_ld16(lane_base + tmem + c, x);
                tmem_ld_wait();
                if (live) {
                    if (c < D) {
                        float4 *dst = reinterpret_cast<float4 *>(a.GM + (cs * D + r) * D + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_float4(__uint_as_float(x[4 * e]), __uint_as_float(x[4 * e + 1]),
                                                 __uint_as_float(x[4 * e + 2]), __uint_as_float(x[4 * e + 3]));
                    } else {
                        a.Gz[cs * D + r] = __uint_as_float(x[0]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}


// the memory update's gradients of one (b, kv head, segment)
template <int D, bool DELTA>
__global__ void __launch_bounds__(192, 1)
k_bwd_update_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const BwdUpdArgs a)
{
    using C = BwdUpdCfg<D>;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int64_t cs = blockIdx.x;                           // chain * S + s
    const int64_t chain = cs / a.S;
    const int s = (int)(cs % a.S);
    const int64_t seg0 = (int64_t)s * a.N;
    const int valid = (int)(a.L - seg0 < a.N ? a.L - seg0 : a.N);
    const int nt = (valid + 127) / 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *sK = smem + C::OFF_K, *sV = smem + C::OFF_V, *sE = smem + C::OFF_E;
    uint8_t *sDU = sK;                                       // -dU / den, after h has read sigma(K)
    uint8_t *sDM = smem + C::OFF_DM, *sM = smem + C::OFF_M;  // hi at +0, lo at +MBYTES
    float *sz = reinterpret_cast<float *>(smem + C::OFF_Z);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars, *mready = bars + 1, *kready = bars + 2, *p12 = bars + 3, *uready = bars + 4;
    uint64_t *p3 = bars + 5, *done = bars + 6, *eready = bars + 7, *hdone = bars + 8;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + C::NBAR * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + C::NBAR * 8 + 4);

    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(mready, 128);
        mbar_init(kready, 128);
        mbar_init(p12, 1);
        mbar_init(uready, 128);
        mbar_init(p3, 1);
        mbar_init(done, 1);
        mbar_init(eready, 128);
        mbar_init(hdone, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (D == 64)       // the padded feature box of sigma(K) stays zero
        for (int i = threadIdx.x; i < C::BOX / 16; i += blockDim.x)
            reinterpret_cast<uint4 *>(sK + C::BOX)[i] = make_uint4(0, 0, 0, 0);
    if (warp == 5) tmem_alloc(tmem_holder, C::TMEM_COLS);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------------------------- loads
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            bool ok = true;
            int issued = 0;
            for (int i = 0; ok && i < nt; ++i) {
                // the tile's buffers are free once the previous tile's last products are done
                if (i > 0 && !(ok = mbar_wait(p3, (i - 1) & 1, abort, WB_P3))) break;
                mbar_arrive_expect_tx(full, 2 * C::NB * C::BOX);
                for (int cb = 0; cb < C::NB; ++cb) {
                    tma_load_3d(sK + cb * C::BOX, &tmK, full, cb * 64, (int)(seg0 + i * 128), (int)chain);
                    tma_load_3d(sV + cb * C::BOX, &tmV, full, cb * 64, (int)(seg0 + i * 128), (int)chain);
                }
                issued = i + 1;
            }
            if (*abort && issued > 0) bwdtc_drain(full, (issued - 1) & 1);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idMN = idesc_bf16(128, D, 0, 1);   // B = dM / M, MN-major
            constexpr uint32_t idK = idesc_bf16(128, D, 0, 0);    // B = dM^T / M^T, K-major
            constexpr uint32_t idH = idesc_bf16(128, 16, 1, 1);   // h: A = sigma(K) MN-major
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aDU = smem_u32(sDU), aE = smem_u32(sE);
            const uint32_t aDM = smem_u32(sDM), aM = smem_u32(sM);
            constexpr uint32_t LO = C::MBYTES;
            bool ok = mbar_wait_short(mready, 0, abort, WB_MF);
            for (int i = 0; ok && i < nt; ++i) {
                if (!(ok = mbar_wait_short(kready, i & 1, abort, WB_FULL))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {                 // dU, sigma(K) M: hi + lo parts
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    const uint64_t ak = sdesc_sw128(aK + off, 16, 1024);
                    mma_ss(tmem + C::T_1, ak, sdesc_sw128(aDM + kk * 2048, C::MBOX, 1024), idMN, kk > 0 ? 1u : 0u);
                    mma_ss(tmem + C::T_1, ak, sdesc_sw128(aDM + LO + kk * 2048, C::MBOX, 1024), idMN, 1u);
                    if (DELTA) {
                        mma_ss(tmem + C::T_2, ak, sdesc_sw128(aM + kk * 2048, C::MBOX, 1024), idMN, kk > 0 ? 1u : 0u);
                        mma_ss(tmem + C::T_2, ak, sdesc_sw128(aM + LO + kk * 2048, C::MBOX, 1024), idMN, 1u);
                    }
                }
                mma_commit(p12);
                if (DELTA) {
                    if (!(ok = mbar_wait_short(eready, i & 1, abort, WB_UR))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)             // h += sigma(K)^T [dden_hi | dden_lo]
                        mma_ss(tmem + C::T_H, sdesc_sw128(aK + kk * 2048, C::BOX, 1024),
                               sdesc_sw128(aE + kk * 2048, C::BOX, 1024), idH, (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(hdone);
                }
                if (!(ok = mbar_wait_short(uready, i & 1, abort, WB_UR))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * C::MBOX + (kk & 3) * 32;
                    // U dM^T, then (-dU / den) M^T into the same accumulator
                    mma_ss(tmem + C::T_3, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(aDM + boff, 16, 1024),
                           idK, kk > 0 ? 1u : 0u);
                    if (DELTA)
                        mma_ss(tmem + C::T_3, sdesc_sw128(aDU + off, 16, 1024), sdesc_sw128(aM + boff, 16, 1024),
                               idK, 1u);
                }
                mma_commit(p3);
            }
            mma_commit(done);
            bwdtc_drain(done, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- rows
        const int r = threadIdx.x;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // dM_s and M_{s-1} as bf16 tiles (row r of each), z_{s-1}
        if (r < D) {
            const float4 *g4 = reinterpret_cast<const float4 *>(a.dMs + (cs * D + r) * D);
            const float4 *m4 = reinterpret_cast<const float4 *>(a.snapM + (cs * D + r) * D);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 8) {
                const int ch = (c0 & 63) >> 3;
                const int off = (c0 >> 6) * C::MBOX + r * 128 + ((ch ^ (r & 7)) << 4);
                // x = hi + lo in two bf16 parts, 8 values at a time
                auto split = [&](const float4 &x0, const float4 &x1, uint8_t *dst) {
                    const float v8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hi[e] = pack_bf16x2(v8[2 * e], v8[2 * e + 1]);
                        lo[e] = pack_bf16x2(v8[2 * e] - __uint_as_float(hi[e] << 16),
                                            v8[2 * e + 1] - __uint_as_float(hi[e] & 0xffff0000u));
                    }
                    *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(dst + C::MBYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                };
                split(g4[c0 / 4], g4[c0 / 4 + 1], sDM);
                if (DELTA) split(m4[c0 / 4], m4[c0 / 4 + 1], sM);
            }
            sz[r] = DELTA ? a.snapZ[cs * D + r] : 0.f;
        }
        fence_proxy_async_smem();
        mbar_arrive(mready);
        const uint64_t one2 = f2_pack(1.f, 1.f);
        const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
        bool ok = mbar_wait(mready, 0, abort, WB_MF);       // z visible to every row
        for (int i = 0; ok && i < nt; ++i) {
            const int t = i * 128 + r;                           // row in the segment
            const bool in = t < valid;
            const uint32_t keep = in ? 0xFFFFFFFFu : 0u;         // rows past the end: sigma = 0
            if (!(ok = mbar_wait(full, i & 1, abort, WB_FULL))) break;
            // sigma(k) over the K row, den = sigma(k) . z from the unrounded sigma
            uint64_t dp2[2] = {0ull, 0ull};
#pragma unroll 4
            for (int c0 = 0; c0 < D; c0 += 8) {
                const int ch = (c0 & 63) >> 3;
                uint4 *ptr = reinterpret_cast<uint4 *>(sK + (c0 >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4));
                const uint4 x = *ptr;
                uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = __uint_as_float(w4[e] << 16), x1 = __uint_as_float(w4[e] & 0xffff0000u);
                    float a0, a1, p0, p1;
                    f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
                    f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
                    const float s0 = __uint_as_float(__float_as_uint(fmaxf(p0, ex2(a0))) & keep);
                    const float s1 = __uint_as_float(__float_as_uint(fmaxf(p1, ex2(a1))) & keep);
                    if (DELTA) dp2[e & 1] = f2_fma(f2_pack(s0, s1), f2_pack(sz[c0 + 2 * e], sz[c0 + 2 * e + 1]), dp2[e & 1]);
                    w4[e] = pack_bf16x2(s0, s1);
                }
                *ptr = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            float d0, d1, d2, d3;
            f2_unpack(dp2[0], d0, d1);
            f2_unpack(dp2[1], d2, d3);
            const float den = (d0 + d1) + (d2 + d3);
            const float inv = den == 0.f ? 0.f : 1.f / den;
            fence_proxy_async_smem();
            mbar_arrive(kready);
            if (!(ok = mbar_wait(p12, i & 1, abort, WB_SDP))) break;
            tc_fence_after();
            const int64_t row = chain * a.L + seg0 + t;
            // dU_t (dv += dU_t) and, delta, R_t = (sigma(k_t) M) / den, U_t = v_t - R_t written
            // over V, -dU_t / den over the dU tile, dden_t = dU_t . R_t / den into the column box
            float dd = 0.f;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t du[32], rm[32];
                tmem_ld32(lane_base + tmem + C::T_1 + c, du);
                if (DELTA) tmem_ld32(lane_base + tmem + C::T_2 + c, rm);
                tmem_ld_wait();
                if (in) {
                    float4 *dvp = reinterpret_cast<float4 *>(a.dv + row * D + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float4 x = dvp[e];
                        x.x += __uint_as_float(du[4 * e]);
                        x.y += __uint_as_float(du[4 * e + 1]);
                        x.z += __uint_as_float(du[4 * e + 2]);
                        x.w += __uint_as_float(du[4 * e + 3]);
                        dvp[e] = x;
                    }
                }
                if (DELTA) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ch = ((c & 63) >> 3) + e;
                        const int off = (c >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4);
                        uint4 *vp = reinterpret_cast<uint4 *>(sV + off);
                        const uint4 vx = *vp;
                        const uint32_t v4[4] = {vx.x, vx.y, vx.z, vx.w};
                        uint32_t u4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int i0 = 8 * e + 2 * u;
                            const float r0 = __uint_as_float(rm[i0]) * inv, r1 = __uint_as_float(rm[i0 + 1]) * inv;
                            dd = fmaf(__uint_as_float(du[i0]), r0, fmaf(__uint_as_float(du[i0 + 1]), r1, dd));
                            u4[u] = pack_bf16x2(__uint_as_float(v4[u] << 16) - r0, __uint_as_float(v4[u] & 0xffff0000u) - r1);
                        }
                        *vp = make_uint4(u4[0], u4[1], u4[2], u4[3]);
                    }
                }
            }
            const float dden = DELTA ? dd * inv : 0.f;
            if (DELTA) {
                // dden as hi + lo columns; sigma(K) stays until h has read it
                uint8_t *ex = sE + r * 128;
                const uint32_t dh = pack_bf16x2(dden, 0.f);
                const uint32_t dl = pack_bf16x2(0.f, dden - __uint_as_float(dh << 16));
                *reinterpret_cast<uint4 *>(ex + ((0 ^ (r & 7)) << 4)) = make_uint4(dh | dl, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(ex + ((1 ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
                fence_proxy_async_smem();
                mbar_arrive(eready);
                // -dU / den over sigma(K) once h has read it (dU read again from TMEM)
                if (!(ok = mbar_wait(hdone, i & 1, abort, WB_UR))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t du[32];
                    tmem_ld32(lane_base + tmem + C::T_1 + c, du);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ch = ((c & 63) >> 3) + e;
                        const int off = (c >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4);
                        uint32_t n4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            n4[u] = pack_bf16x2(-__uint_as_float(du[8 * e + 2 * u]) * inv,
                                                -__uint_as_float(du[8 * e + 2 * u + 1]) * inv);
                        *reinterpret_cast<uint4 *>(sDU + off) = make_uint4(n4[0], n4[1], n4[2], n4[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(uready);
            if (!(ok = mbar_wait(p3, i & 1, abort, WB_P3))) break;
            tc_fence_after();
            // dsigma(k_t) = U dM^T - (dU / den) M^T + dden z (without the dz_s term)
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t x[32];
                tmem_ld32(lane_base + tmem + C::T_3 + c, x);
                tmem_ld_wait();
                if (in) {
                    float4 *dst = reinterpret_cast<float4 *>(a.dsk + row * D + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(fmaf(dden, sz[c + 4 * e], __uint_as_float(x[4 * e])),
                                             fmaf(dden, sz[c + 4 * e + 1], __uint_as_float(x[4 * e + 1])),
                                             fmaf(dden, sz[c + 4 * e + 2], __uint_as_float(x[4 * e + 2])),
                                             fmaf(dden, sz[c + 4 * e + 3], __uint_as_float(x[4 * e + 3])));
                }
            }
        }
        // h_s: lane a of the h accumulator is key feature a
        if (ok && mbar_wait(done, 0, abort, WB_DONE)) {
            tc_fence_after();
            uint32_t x[16];
            tmem_ld16(lane_base + tmem + C::T_H, x);
            tmem_ld_wait();
            if (r < D) a.h[cs * D + r] = DELTA ? __uint_as_float(x[0]) + __uint_as_float(x[1]) : 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace infini
