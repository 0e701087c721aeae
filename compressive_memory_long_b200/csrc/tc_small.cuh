// Fused Infini-attention forward for 64-token segments and the additive memory rule, one
// launch for the whole problem (sm_100a).
//
// The additive update (AI Wiki "Infini-Attention", "How does the compressive memory
// work?") makes M_{s-1} = M0 + sum_{j<s} sigma(K_j)^T V_j a prefix sum ("What is linear
// attention and the delta rule?"), so segments can be processed in parallel once each
// knows the sum of its predecessors.  One CTA owns a unit of two consecutive segments
// (128 tokens) of one head and:
//   1. loads Q, K, V of the unit with TMA and forms sigma(K), sigma(Q) in shared memory;
//   2. on the tensor cores: S = Q K^T over the unit (a 128 x 128 tile whose block-diagonal
//      causal mask keeps each segment to its own keys, "What happens inside the
//      Infini-attention block?"), and the per-segment increments
//      [dM_s | dz_s] = sigma(K_s)^T [V_s | 1];
//   3. publishes its aggregate dM_0 + dM_1 and finds the exclusive prefix M_start: with few
//      units per head ("direct" mode) by summing M0 and every earlier aggregate itself, else
//      with a single-pass decoupled look-back over earlier units of the same head (Merrill
//      and Garland, "Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016): a
//      predecessor's inclusive prefix ends the walk, its aggregate continues it;
//   4. softmax and O = P V, then R_0 = sigma(Q) M_start and R_1 = sigma(Q) (M_start + dM_0)
//      (rows of the first segment read R_0, rows of the second R_1), and the gated output.
// Units take tickets in start order, so a CTA only waits for units that started before it
// (running or finished): no unit waits on one that cannot run.  Every wait is bounded.
// Layout limits: bf16, d = 64, N = 64, L % 128 == 0.  With several query heads per key/value
// head each query head is a chain of its own (its own units, flags and published states);
// keys, values, M0 and z0 are read through the head's key/value head, and the first query
// head of a group writes M_out and z_out.
#pragma once

#include "tc_common.cuh"

namespace infini {
namespace tc {

struct SmallCfg {
    static constexpr int D = 64, TOK = 128, SEG = 64;
    static constexpr int BOX = 128 * 128;          // 128 rows x 64 bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + BOX;
    static constexpr int OFF_V = OFF_K + BOX;      // V box, then a constant box (col 0 = 1)
    static constexpr int OFF_SK = OFF_V + 2 * BOX; // sigma(K): features padded to 128
    static constexpr int OFF_SQ = OFF_SK + 2 * BOX;
    static constexpr int MB = 64 * 128;            // 64 key rows x 64 bf16 values
    static constexpr int OFF_M0 = OFF_SQ + BOX;
    static constexpr int OFF_M1 = OFF_M0 + MB;
    static constexpr int OFF_Z = OFF_M1 + MB;      // z_start[64], z_mid[64] (fp32)
    static constexpr int ROW = 68;                 // floats per state row: 64 M, z, 3 pad
    static constexpr int STATE = 64 * ROW;         // floats of one [64][ROW] state
    static constexpr int STATE4 = STATE / 4;       // float4s of one state (1088)
    static constexpr int OFF_AGG = OFF_Z + 2 * 64 * 4;   // this unit's aggregate [64][ROW]
    static constexpr int OFF_D0 = OFF_AGG + STATE * 4;   // first segment's increment
    static constexpr int OFF_EX = OFF_D0 + STATE * 4;    // exclusive prefix
    static constexpr int OFF_BAR = OFF_EX + STATE * 4;
    static constexpr int NBAR = 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 32;
    static constexpr int ALLOC = BYTES + 1024;
};

struct SmallArgs {
    const float *beta;
    const float *M0, *z0;          // may be NULL
    __nv_bfloat16 *out;
    float *M_out, *z_out;
    int *ticket;                   // zeroed before the launch
    int *m0_done;                  // [chains] units that have read M0 (direct mode), zeroed
    int *flags;                    // [chains * U], zeroed before the launch
    float *agg, *incl;             // [chains * U, 64, ROW]
    int64_t L;
    int U, H, Hkv;
    int chains;                    // query heads, B * H
    int direct;                    // 1: every unit sums M0 and all earlier aggregates itself
    int in_place;                  // 1: M_out / z_out are the very buffers M0 / z0 (H == Hkv)
};

// the key/value head of query-head chain c = b * H + h
__device__ __forceinline__ int64_t kv_chain(int64_t c, int H, int Hkv)
{
    return (c / H) * Hkv + (c % H) / (H / Hkv);
}

enum : int { FLAG_AGG = 1, FLAG_INCL = 2 };
enum : int { WS_FULL = 501, WS_S = 502, WS_SIG = 503, WS_D = 504, WS_P = 505, WS_O = 506,
             WS_M = 507, WS_R = 508, WS_LOOK = 509, WS_DRAIN = 510 };

__device__ __forceinline__ void small_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WS_DRAIN);
            return;
        }
    }
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float sigma_s(float x) { return elu1(x); }

// Named barrier 1 over the 128 work threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_or_128(bool v)
{
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)v)
        : "memory");
    return out != 0;
}


__device__ __forceinline__ void tmem_st16_s(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__global__ void __launch_bounds__(256, 1)
k_small_linear_fused(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const SmallArgs a)
{
    using C = SmallCfg;
    constexpr int D = C::D;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint8_t *sQ = smem + C::OFF_Q, *sK = smem + C::OFF_K, *sV = smem + C::OFF_V;
    uint8_t *sSK = smem + C::OFF_SK, *sSQ = smem + C::OFF_SQ;
    uint8_t *sM0 = smem + C::OFF_M0, *sM1 = smem + C::OFF_M1;
    float *sZ0 = reinterpret_cast<float *>(smem + C::OFF_Z), *sZ1 = sZ0 + 64;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars, *s_done = bars + 1, *sig_ready = bars + 2, *d_done = bars + 3;
    uint64_t *p_ready = bars + 4, *o_done = bars + 5, *m_ready = bars + 6, *r_done = bars + 7;
    uint64_t *mma_done = bars + 8;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    volatile int *s_ticket = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
    volatile int *s_state = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 12);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        *s_ticket = atomicAdd(a.ticket, 1);
        mbar_init(full, 1);
        mbar_init(s_done, 1);
        mbar_init(sig_ready, 128);
        mbar_init(d_done, 1);
        mbar_init(p_ready, 128);
        mbar_init(o_done, 1);
        mbar_init(m_ready, 128);
        mbar_init(r_done, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        *s_state = 0;
        fence_barrier_init();
        // this thread knows its unit already: start the loads before the TMEM allocation
        // and the block barrier, so they overlap both
        const int t0 = *s_ticket;
        const int64_t ch = t0 % a.chains;
        const int64_t kvc = kv_chain(ch, a.H, a.Hkv);
        const int un = t0 / a.chains;
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_arrive_expect_tx(full, 3 * C::BOX);
        tma_load_3d(sQ, &tmQ, full, 0, un * C::TOK, (int)ch);
        tma_load_3d(sK, &tmK, full, 0, un * C::TOK, (int)kvc);
        tma_load_3d(sV, &tmV, full, 0, un * C::TOK, (int)kvc);
    }
    if (warp == 1) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_S = tmem, T_O = tmem + 128, T_R0 = tmem + 192, T_R1 = tmem + 256;
    const uint32_t T_D0 = tmem + 320, T_D1 = tmem + 400;
    // tickets interleave heads (unit-major), so every head advances side by side
    const int t = *s_ticket;
    const int64_t chain = t % a.chains;     // = b * H + h
    const int64_t kvc = kv_chain(chain, a.H, a.Hkv);
    const bool state_writer = (chain % a.H) % (a.H / a.Hkv) == 0;   // first query head of its group
    const int unit = t / a.chains;
    const int64_t idx = chain * a.U + unit;

    if (warp == 0) {
        if (lane == 0 && *abort) small_drain(full, 0);   // the loads were issued above
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idD = idesc_bf16(128, D + 16, 1, 1);
            constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            const uint32_t aSK = smem_u32(sSK), aSQ = smem_u32(sSQ);
            const uint32_t aM0 = smem_u32(sM0), aM1 = smem_u32(sM1);
            bool ok = mbar_wait_short(full, 0, abort, WS_FULL);
            if (ok) {   // S = Q K^T over the unit
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(T_S, sdesc_sw128(aQ + kk * 32, 16, 1024), sdesc_sw128(aK + kk * 32, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                mma_commit(s_done);
            }
            if (ok) ok = mbar_wait_short(sig_ready, 0, abort, WS_SIG);
            if (ok) {   // [dM_s | dz_s] = sigma(K_s)^T [V_s | 1], s = first and second segment
                tc_fence_after();
#pragma unroll
                for (int seg = 0; seg < 2; ++seg)
#pragma unroll
                    for (int kk = 0; kk < C::SEG / 16; ++kk) {
                        const uint32_t off = (seg * C::SEG + kk * 16) * 128;
                        mma_ss(seg ? T_D1 : T_D0, sdesc_sw128(aSK + off, C::BOX, 1024),
                               sdesc_sw128(aV + off, C::BOX, 1024), idD, kk > 0 ? 1u : 0u);
                    }
                mma_commit(d_done);
            }
            if (ok) ok = mbar_wait_short(p_ready, 0, abort, WS_P);
            if (ok) {   // O = P V
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C::TOK / 16; ++kk)
                    mma_ts(T_O, T_S + kk * 8, sdesc_sw128(aV + kk * 2048, C::BOX, 1024), idO,
                           kk > 0 ? 1u : 0u);
                mma_commit(o_done);
            }
            if (ok) ok = mbar_wait_short(m_ready, 0, abort, WS_M);
            if (ok) {   // R_0 = sigma(Q) M_start, R_1 = sigma(Q) M_mid
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    mma_ss(T_R0, sdesc_sw128(aSQ + kk * 32, 16, 1024),
                           sdesc_sw128(aM0 + kk * 2048, C::MB, 1024), idO, kk > 0 ? 1u : 0u);
                    mma_ss(T_R1, sdesc_sw128(aSQ + kk * 32, 16, 1024),
                           sdesc_sw128(aM1 + kk * 2048, C::MB, 1024), idO, kk > 0 ? 1u : 0u);
                }
                mma_commit(r_done);
            }
            mma_commit(mma_done);
            small_drain(mma_done, 0);
        }
    } else if (warp >= 4) {
        const int r = threadIdx.x - 128;                 // row: token of the unit / feature
        const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
        // constants: the box after V has column 0 = 1; the padded half of sigma(K) is 0
        for (int i = r; i < 128 * 8; i += 128) {
            const int row = i / 8, ch = i % 8;
            *reinterpret_cast<uint4 *>(sV + C::BOX + row * 128 + ((ch ^ (row & 7)) << 4)) =
                make_uint4(ch == 0 ? 0x3F80u : 0u, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sSK + C::BOX + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
        float *sAgg = reinterpret_cast<float *>(smem + C::OFF_AGG);
        float *sD0 = reinterpret_cast<float *>(smem + C::OFF_D0);
        float *sEx = reinterpret_cast<float *>(smem + C::OFF_EX);
        // bf16 row r, same swizzle.  Not unrolled: the kernel runs its code once per CTA, so
        // fewer distinct instructions (instruction-cache misses) matter more than loop overhead.
        auto sigma_row = [&](const uint8_t *src, uint8_t *dst) {
#pragma unroll 1
            for (int ch = 0; ch < 8; ++ch) {
                const int o = r * 128 + ((ch ^ (r & 7)) << 4);
                const uint4 x = *reinterpret_cast<const uint4 *>(src + o);
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 t2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                    w[e] = pack_bf16x2(sigma_s(__low2float(t2)), sigma_s(__high2float(t2)));
                }
                *reinterpret_cast<uint4 *>(dst + o) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        };
        float l = 0.f;                  // softmax row sum
        bool ok = mbar_wait_short(full, 0, abort, WS_FULL);
        if (ok) {                       // sigma(K) first: the increment MMAs need only it
            sigma_row(sK, sSK);
            fence_proxy_async_smem();
            mbar_arrive(sig_ready);
        }
        // ---- this unit's increments into shared memory: D0 (first segment), D0 + D1
        if (ok) ok = mbar_wait_short(d_done, 0, abort, WS_D);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < 80; c0 += 16) {
                uint32_t x[16], y[16];
                tmem_ld16(lane_base + T_D0 + c0, x);
                tmem_ld16(lane_base + T_D1 + c0, y);
                tmem_ld_wait();
                if (r < D) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int col = c0 + e;
                        if (col < C::ROW) {
                            const float x0 = __uint_as_float(x[e]);
                            sD0[r * C::ROW + col] = x0;
                            sAgg[r * C::ROW + col] = x0 + __uint_as_float(y[e]);
                        }
                    }
                }
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // publish the aggregate (coalesced 16-byte stores by all 128 threads)
        if (ok && (unit > 0 || a.direct)) {
            float4 *dst = reinterpret_cast<float4 *>(a.agg + idx * C::STATE);
            const float4 *src = reinterpret_cast<const float4 *>(sAgg);
            for (int i = r; i < C::STATE4; i += 128) dst[i] = src[i];
            __threadfence();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // Unit 0 of a long head publishes no aggregate, only its inclusive prefix: every other
        // walk then ends at an inclusive prefix, and only unit 0 reads M0 / z0 -- which M_out /
        // z_out (written by the last unit, after its walk) may alias.
        // (a test hook can make unit 0 withhold its publishes: the later units' waits run out)
        const bool withhold = unit == 0 && g_test_withhold != 0;
        if (ok && r == 0 && (unit > 0 || a.direct) && !withhold) st_release_gpu(a.flags + idx, FLAG_AGG);

        // the local softmax and sigma(Q) come after the aggregate is published: later units
        // of the head wait for it, while this unit's own softmax is not on their path
        // ---- local softmax: row r sees the 64 keys of its own segment, up to itself
        if (ok) ok = mbar_wait_short(s_done, 0, abort, WS_S);
        if (ok) {
            tc_fence_after();
            const int lo = (r >> 6) << 6;                // first key of this row's segment
            uint32_t v[2][32];
            tmem_ld32(lane_base + T_S + lo, v[0]);
            tmem_ld32(lane_base + T_S + lo + 32, v[1]);
            tmem_ld_wait();
            float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if (lo + c * 32 + e > r) v[c][e] = __float_as_uint(-INFINITY);
                    pm[e & 3] = fmaxf(pm[e & 3], __uint_as_float(v[c][e]));
                }
            const float mt = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
            const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
            const float mk = mt * kscale;
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t zero16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) zero16[e] = 0u;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2(fmaf(__uint_as_float(v[c][2 * e]), kscale, -mk));
                    const float p1 = ex2(fmaf(__uint_as_float(v[c][2 * e + 1]), kscale, -mk));
                    ps[e & 3] += p0 + p1;
                    pk[e] = pack_bf16x2(p0, p1);
                }
                // P over the S columns: this segment's keys, and zeros for the other segment
                tmem_st16_s(lane_base + T_S + (lo >> 1) + c * 16, pk);
                tmem_st16_s(lane_base + T_S + ((64 - lo) >> 1) + c * 16, zero16);
            }
            l = (ps[0] + ps[1]) + (ps[2] + ps[3]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_ready);
        }
        if (ok) sigma_row(sQ, sSQ);    // sigma(Q) for the retrieval, off the critical path

        // ---- exclusive prefix of this unit, kept as float4 per thread (i = r + 128 k)
        constexpr int KQ = (C::STATE4 + 127) / 128;
        float4 ex[KQ];
#pragma unroll
        for (int k = 0; k < KQ; ++k) ex[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        auto add_state = [&](const float *base) {
            const float4 *src = reinterpret_cast<const float4 *>(base);
#pragma unroll
            for (int k = 0; k < KQ; ++k) {
                const int i = r + 128 * k;
                if (i < C::STATE4) {
                    const float4 x = __ldcg(src + i);
                    ex[k].x += x.x; ex[k].y += x.y; ex[k].z += x.z; ex[k].w += x.w;
                }
            }
        };
        auto add_initial = [&]() {      // M0 and z0 into the [64][ROW] layout
#pragma unroll
            for (int k = 0; k < KQ; ++k) {
                const int i = r + 128 * k;
                if (i < C::STATE4) {
                    const int row = i / (C::ROW / 4), c4 = i % (C::ROW / 4);
                    if (c4 < D / 4) {
                        if (a.M0) {
                            const float4 m = *reinterpret_cast<const float4 *>(a.M0 + (kvc * D + row) * D + 4 * c4);
                            ex[k].x += m.x; ex[k].y += m.y; ex[k].z += m.z; ex[k].w += m.w;
                        }
                    } else if (a.z0) {
                        ex[k].x += a.z0[kvc * D + row];
                    }
                }
            }
        };
        if (a.direct) {
            // wait until every earlier unit of the head has published its aggregate: thread j
            // watches unit j, so the flags are polled side by side (unit < 64 <= 128 here)
            bool bad = false;
            if (ok && r < unit) {
                const int *fp = a.flags + chain * a.U + r;
                const long long t0 = clock64();
                while (ld_acquire_gpu(fp) == 0) {
                    if (clock64() - t0 > spin_limit() || wait_status_set()) {
                        atomicCAS(&g_wait_status, 0, WS_LOOK);
                        bad = true;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            if (bar_or_128(bad) && ok) {
                ok = false;
                *abort = 1;
            }
            if (ok) {
                for (int j = 0; j < unit; ++j) add_state(a.agg + (chain * a.U + j) * C::STATE);
                add_initial();
            }
            // in place, the last unit may overwrite M0 / z0 only after every other unit of
            // the head has read them
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ok && r == 0 && a.in_place) {
                __threadfence();
                if (unit + 1 < a.U) {
                    atomicAdd(a.m0_done + chain, 1);
                } else {
                    const long long t0 = clock64();
                    while (ld_acquire_gpu(a.m0_done + chain) < a.U - 1) {
                        if (clock64() - t0 > spin_limit() || wait_status_set()) {
                            atomicCAS(&g_wait_status, 0, WS_LOOK);
                            *s_state = -1;
                            break;
                        }
                        __nanosleep(32);
                    }
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ok && unit + 1 == a.U && *s_state < 0) {
                ok = false;
                *abort = 1;
            }
        } else {
            for (int j = unit - 1; ok && j >= 0; --j) {
                if (r == 0) {
                    const int *fp = a.flags + chain * a.U + j;
                    int f = ld_acquire_gpu(fp);
                    const long long t0 = clock64();
                    while (f == 0) {
                        if (clock64() - t0 > spin_limit() || wait_status_set()) {
                            atomicCAS(&g_wait_status, 0, WS_LOOK);
                            f = -1;
                            break;
                        }
                        __nanosleep(32);
                        f = ld_acquire_gpu(fp);
                    }
                    *s_state = f;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                const int f = *s_state;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (f < 0) {
                    ok = false;
                    *abort = 1;
                    break;
                }
                add_state((f == FLAG_INCL ? a.incl : a.agg) + (chain * a.U + j) * C::STATE);
                if (f == FLAG_INCL) break;
            }
            if (ok && unit == 0) add_initial();
        }
        if (ok) {
            float4 *sEx4 = reinterpret_cast<float4 *>(sEx);
            const float4 *sAgg4 = reinterpret_cast<const float4 *>(sAgg);
#pragma unroll
            for (int k = 0; k < KQ; ++k) {
                const int i = r + 128 * k;
                if (i < C::STATE4) {
                    sEx4[i] = ex[k];
                    if (unit + 1 == a.U && state_writer) {  // the head's final state
                        const float4 g = sAgg4[i];
                        const int row = i / (C::ROW / 4), c4 = i % (C::ROW / 4);
                        if (c4 < D / 4)
                            reinterpret_cast<float4 *>(a.M_out + (kvc * D + row) * D)[c4] =
                                make_float4(ex[k].x + g.x, ex[k].y + g.y, ex[k].z + g.z, ex[k].w + g.w);
                        else
                            a.z_out[kvc * D + row] = ex[k].x + g.x;
                    }
                    if (!a.direct && unit + 1 < a.U) {      // inclusive prefix for successors
                        const float4 g = sAgg4[i];
                        reinterpret_cast<float4 *>(a.incl + idx * C::STATE)[i] =
                            make_float4(ex[k].x + g.x, ex[k].y + g.y, ex[k].z + g.z, ex[k].w + g.w);
                    }
                }
            }
            if (!a.direct && unit + 1 < a.U) __threadfence();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok) {
            if (r == 0 && !a.direct && unit + 1 < a.U && !withhold) st_release_gpu(a.flags + idx, FLAG_INCL);
            if (r < D) {
                const float *exr = sEx + r * C::ROW, *d0r = sD0 + r * C::ROW;
                // M_start and M_mid rows (key r) as bf16 B operands, z as fp32
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t w0[4], w1[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = ch * 8 + 2 * e;
                        w0[e] = pack_bf16x2(exr[q], exr[q + 1]);
                        w1[e] = pack_bf16x2(exr[q] + d0r[q], exr[q + 1] + d0r[q + 1]);
                    }
                    const int o = r * 128 + ((ch ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4 *>(sM0 + o) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                    *reinterpret_cast<uint4 *>(sM1 + o) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                }
                sZ0[r] = exr[D];
                sZ1[r] = exr[D] + d0r[D];
            }
            fence_proxy_async_smem();
            mbar_arrive(m_ready);
        }
        // ---- epilogue: gate the local and memory reads of row r
        if (ok) ok = mbar_wait_short(o_done, 0, abort, WS_O);
        if (ok) ok = mbar_wait_short(r_done, 0, abort, WS_R);
        if (ok) {
            tc_fence_after();
            asm volatile("bar.sync 1, 128;" ::: "memory");   // every row's z is in place
            const float *zz = (r < C::SEG) ? sZ0 : sZ1;
            float den = 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {    // sigma(q) . z from the bf16 sigma(Q) row
                const uint4 qv = *reinterpret_cast<const uint4 *>(sSQ + r * 128 + ((ch ^ (r & 7)) << 4));
                uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 t2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
                    den = fmaf(__low2float(t2), zz[ch * 8 + 2 * e], den);
                    den = fmaf(__high2float(t2), zz[ch * 8 + 2 * e + 1], den);
                }
            }
            const int h = (int)(chain % a.H);
            const float g = 1.f / (1.f + __expf(-a.beta[h]));
            const float wl = (1.f - g) / l;
            const float wm = den == 0.f ? 0.f : g / den;
            const uint32_t tR = (r < C::SEG) ? T_R0 : T_R1;   // uniform per warp
            __nv_bfloat16 *orow = a.out + (chain * a.L + (int64_t)unit * C::TOK + r) * D;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t o[32], rr[32];
                tmem_ld32(lane_base + T_O + c, o);
                tmem_ld32(lane_base + tR + c, rr);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(fmaf(__uint_as_float(rr[2 * e]), wm, __uint_as_float(o[2 * e]) * wl),
                                        fmaf(__uint_as_float(rr[2 * e + 1]), wm, __uint_as_float(o[2 * e + 1]) * wl));
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
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
