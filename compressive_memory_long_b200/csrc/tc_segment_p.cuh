// Fused Infini-attention segment kernel, persistent form (sm_100a).
//
// Same arithmetic as tc_segment.cuh (AI Wiki "Infini-Attention", "What happens inside the
// Infini-attention block?"): per query row, causal softmax attention over the keys of its
// segment, the retrieval sigma(q) M_{s-1} / (sigma(q) . z_{s-1}) and the sigmoid gate.
//
// Work item: the query tiles A = 2p and B = 2p + 1 (128 rows each) of one (b, h, segment);
// both read the same K/V tiles, loaded once.  Tile B needs key tiles 0..2p+1, tile A 0..2p.
// One CTA per SM walks a static list of units; a unit is the pair of items p and
// npairs - 1 - p of one (b, h, segment) (heavier first), so every unit costs the same
// number of key steps and the list balances without a work counter.  Consecutive units are
// the pairs of one segment, so the CTAs that run at the same time share its keys in L2.
//
// Roles: softmax warpgroups A (warps 0-3) and B (warps 4-7) in ping-pong with the tensor
// core; TMA producer (warp 8); MMA issuer (warp 9); warps 10-11 only lend their registers
// (setmaxnreg).  TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+d),
// O_B [256+d, 256+2d).  P (bf16) is written over the first 64 columns of its own S tile;
// tcgen05.mma operations execute in issue order, so P is read before the next S overwrites
// it.  After the last P V of a tile the retrieval R_X = sigma(Q_X) M_{s-1} reuses S_X.
//
// Epilogue: each softmax thread writes its gated output row into a staging buffer in the
// 128-byte-swizzled layout of a Q tile and one thread writes the tile with a TMA store
// (full 128-byte lines instead of one 16-byte piece per row and instruction).  Tile A stages
// in its own Q buffer, tile B in M's buffer at d = 128 (free once R_B has read it; at d = 64
// M's buffer is too small and tile B stages in its Q buffer).  z_{s-1} arrives in shared
// memory with M (one bulk copy on the same barrier).  Each item's Q tiles are prefetched
// into L2 when the producer reaches the item, so their loads, which wait for the buffers,
// land from L2.
//
// Across items: the producer loads the next item's keys and values as soon as ring stages
// free up, Q_A once tile A's output store has read its buffer, Q_B once R_B has read
// sigma(Q_B), M and z once tile B's store has read M's buffer; the issuer starts the next
// item's S_X once warpgroup X has read O_X and R_X (epi_done), so the next item's loads and
// first scores overlap the current item's tail.  All waits are bounded (tc_common.cuh).
#pragma once

#include "tc_common.cuh"
#include "tc_segment.cuh"

namespace infini {
namespace tc {

template <int D>
struct SegPCfg {
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
    static constexpr int OFF_Z = OFF_M + MBYTES;       // z_{s-1}, fp32, loaded with M
    // q_full[2], m_full, k_full/v_full/kv_empty[ST],
    // s_full/p_full/sq_full/r_full/epi_done/st_ready/out_free[2], mma_done
    static constexpr int NBAR = 3 + 3 * STAGES + 2 * 7 + 1;
    static constexpr int OFF_BAR = OFF_Z + D * 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
    // the output tile of a query tile is staged in shared memory and written by one TMA store:
    // tile A through its Q buffer, tile B through M's buffer when it holds a tile (d = 128:
    // Q_B of the next item need not wait for the store), else through its own Q buffer
    static constexpr bool B_OUT_IN_M = MBYTES >= TILE;
};

// wait ids recorded in g_wait_status
enum : int { WT_KV_EMPTY = 401, WT_Q = 402, WT_K = 403, WT_P = 404, WT_V = 405, WT_S = 406,
             WT_R = 407, WT_M = 408, WT_SQ = 409, WT_EPI = 410, WT_QFREE = 411, WT_DRAIN = 412,
             WT_STAGED = 413, WT_MFREE = 414 };

__device__ __forceinline__ void segp_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WT_DRAIN);
            return;
        }
    }
}

// The static work list.  Unit u = (group, j): group = (b*H + h) * S + s, j < ceil(npairs/2);
// its items are p = npairs-1-j and, when different, p = j.  Items whose first row lies past
// L (the short last segment) are skipped.  Every role walks the same list.
struct SegPList {
    uint32_t u;    // current unit (fewer than 2^31 units: the host checks)
    int half;      // 0: its heavier item next, 1: its lighter one
    __device__ bool next(const SegArgs &a, uint32_t units, int &p, int &s, int64_t &bh)
    {
        const uint32_t npairs = (uint32_t)a.N >> 8, nu = (npairs + 1) >> 1;
        while (u < units) {
            const uint32_t g = u / nu;
            const uint32_t j = u - g * nu;
            const int pp = (int)(half == 0 ? npairs - 1 - j : j);
            const bool exists = half == 0 || j < npairs - 1 - j;
            if (half == 0) {
                half = 1;
            } else {
                half = 0;
                u += gridDim.x;
            }
            if (!exists) continue;
            const uint32_t bb = g / (uint32_t)a.S;
            const int ss = (int)(g - bb * (uint32_t)a.S);
            if ((int64_t)ss * a.N + pp * 256 >= a.L) continue;
            p = pp;
            s = ss;
            bh = bb;
            return true;
        }
        return false;
    }
};

// An address the compiler must treat as unknown: the issuer builds each descriptor where it
// is used instead of keeping one per stage and k-step live across the item loop.
__device__ __forceinline__ uint32_t opaque_u32(uint32_t x)
{
    asm volatile("" : "+r"(x));
    return x;
}

// sigma(x) = ELU(x) + 1 over the columns [C0, C1) of row r of a Q tile in shared memory
// (128-byte swizzle, 64-column boxes), written back in place as bf16 (max(x + 1, e^min(x, 0))
// on packed fp32 pairs, rounded once); returns sigma(q) . z over those columns in fp32.
template <int C0, int C1, int UNROLL>
__device__ __forceinline__ float segp_sigma_row(uint8_t *q, int r, const float *sZ)
{
    constexpr int BOX = 128 * 128;
    const uint64_t one2 = f2_pack(1.f, 1.f);
    const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
    const float4 *z4 = reinterpret_cast<const float4 *>(sZ);
    uint64_t dp2[2] = {0ull, 0ull};
#pragma unroll UNROLL
    for (int c0 = C0; c0 < C1; c0 += 8) {
        const int ch = (c0 & 63) >> 3;
        uint4 *ptr = reinterpret_cast<uint4 *>(q + (c0 >> 6) * BOX + r * 128 + ((ch ^ (r & 7)) << 4));
        const uint4 qv = *ptr;
        const float4 za = z4[c0 >> 2], zb = z4[(c0 >> 2) + 1];
        const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
        uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
            float a0, a1, p0, p1;
            f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
            f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
            const float s0 = fmaxf(p0, ex2(a0)), s1 = fmaxf(p1, ex2(a1));
            dp2[e & 1] = f2_fma(f2_pack(s0, s1), f2_pack(zz[2 * e], zz[2 * e + 1]), dp2[e & 1]);
            w[e] = pack_bf16x2(s0, s1);
        }
        *ptr = make_uint4(w[0], w[1], w[2], w[3]);
    }
    float d0, d1, d2, d3;
    f2_unpack(dp2[0], d0, d1);
    f2_unpack(dp2[1], d2, d3);
    return (d0 + d1) + (d2 + d3);
}

template <int D>
__global__ void __launch_bounds__(384, 1)
k_segment_tcp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM,
              const __grid_constant__ CUtensorMap tmO, const SegArgs a, const uint32_t units)
{
    using C = SegPCfg<D>;
    constexpr int ST = C::STAGES;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = a.H / a.Hkv;
    uint8_t *sQ[2] = {smem + C::OFF_QA, smem + C::OFF_QB};
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sM = smem + C::OFF_M;
    float *sZ = reinterpret_cast<float *>(smem + C::OFF_Z);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars, *m_full = bars + 2;
    uint64_t *k_full = bars + 3, *v_full = k_full + ST, *kv_empty = v_full + ST;
    uint64_t *s_full = kv_empty + ST, *p_full = s_full + 2, *sq_full = p_full + 2;
    uint64_t *r_full = sq_full + 2, *epi_done = r_full + 2, *st_ready = epi_done + 2;
    uint64_t *out_free = st_ready + 2, *mma_done = out_free + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(q_full + 0, 1);
        mbar_init(q_full + 1, 1);
        mbar_init(m_full, 1);
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(kv_empty + i, 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + x, 1);
            mbar_init(p_full + x, 128);
            mbar_init(sq_full + x, 128);
            mbar_init(r_full + x, 1);
            mbar_init(epi_done + x, 128);
            mbar_init(st_ready + x, 128);
            mbar_init(out_free + x, 1);
        }
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 9) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t T_S[2] = {tmem, tmem + 128};
    const uint32_t T_O[2] = {tmem + 256, tmem + 256 + D};

    SegPList list{blockIdx.x, 0};
    int p, s;
    int64_t bh;

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LOW));
      if (warp == 8) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmM);
            int it = 0, nm = 0;                  // items begun; M loads issued
            int nq[2] = {0, 0};                  // Q_A / Q_B loads issued
            int64_t g = 0;                       // key/value tiles issued so far
            bool ok = true;
            while (ok && list.next(a, units, p, s, bh)) {
                const int64_t chain = (bh / a.H) * a.Hkv + (bh % a.H) / group;
                const int nB = 2 * p + 2;
                const int q_row = s * a.N + p * 256;
                // the item's Q tiles into L2 now (its loads wait for the previous item's
                // buffers; from L2 they then land quickly)
                for (int x = 0; x < 2; ++x)
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_prefetch_l2_3d(&tmQ, cb * 64, q_row + x * 128, (int)bh);
                for (int j = 0; ok && j < nB; ++j) {
                    const int st = (int)(g % ST);
                    if (g >= ST && !(ok = mbar_wait_short(kv_empty + st, (uint32_t)((g / ST) - 1) & 1,
                                                          abort, WT_KV_EMPTY)))
                        break;
                    mbar_arrive_expect_tx(k_full + st, C::TILE);
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d(sK + st * C::TILE + cb * C::BOX, &tmK, k_full + st, cb * 64,
                                    s * a.N + j * 128, (int)chain);
                    mbar_arrive_expect_tx(v_full + st, C::TILE);
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d(sV + st * C::TILE + cb * C::BOX, &tmV, v_full + st, cb * 64,
                                    s * a.N + j * 128, (int)chain);
                    ++g;
                    if (j > 1) continue;
                    // after the first key/value tile Q_A, whose buffer holds tile A's staged
                    // output of the previous item until its store has read it; after the
                    // second Q_B, free once R_B has read sigma(Q_B) (or, when tile B's output
                    // goes through sQ[1], once that store has read it)
                    uint64_t *gate = j == 0 ? out_free + 0 : (C::B_OUT_IN_M ? r_full + 1 : out_free + 1);
                    if (it > 0 && !(ok = mbar_wait(gate, (it - 1) & 1, abort, WT_QFREE))) break;
                    mbar_arrive_expect_tx(q_full + j, C::TILE);
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d(sQ[j] + cb * C::BOX, &tmQ, q_full + j, cb * 64, q_row + j * 128, (int)bh);
                    ++nq[j];
                }
                // M_{s-1} and z_{s-1}, needed only by the item's retrieval: sM is free once
                // R_B has read it (or, when tile B's output goes through sM, once that store
                // has read it)
                if (ok && it > 0)
                    ok = mbar_wait(C::B_OUT_IN_M ? out_free + 1 : r_full + 1, (it - 1) & 1, abort, WT_MFREE);
                if (ok) {
                    mbar_arrive_expect_tx(m_full, C::MBYTES + D * 4);
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d(sM + cb * C::MBOX, &tmM, m_full, cb * 64, 0, (int)(chain * a.S + s));
                    bulk_load(sZ, a.snapZ + (chain * a.S + s) * (int64_t)D, D * 4, m_full);
                    ++nm;
                }
                ++it;
            }
            if (*abort) {
                // let every copy this thread issued land before the CTA exits: the last Q_A,
                // Q_B and M, the last ST key/value tiles (older tiles completed before their
                // stage was reused)
                for (int x = 0; x < 2; ++x)
                    if (nq[x] > 0) segp_drain(q_full + x, (uint32_t)(nq[x] - 1) & 1);
                if (nm > 0) segp_drain(m_full, (uint32_t)(nm - 1) & 1);
                for (int64_t t = (g > ST ? g - ST : 0); t < g; ++t) {
                    segp_drain(k_full + t % ST, (uint32_t)(t / ST) & 1);
                    segp_drain(v_full + t % ST, (uint32_t)(t / ST) & 1);
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
            int it = 0;
            int64_t g = 0;                       // key/value tiles consumed so far
            uint32_t np[2] = {0u, 0u};           // P phases consumed so far per tile
            bool ok = true;

            auto issue_s = [&](int x, int64_t t) {
                const uint32_t kbase = opaque_u32(aK + (uint32_t)(t % ST) * C::TILE);
                const uint32_t qbase = opaque_u32(aQ[x]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(T_S[x], sdesc_sw128(qbase + off, 16, 1024),
                           sdesc_sw128(kbase + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + x);
            };
            // O_X += P_X(i) V(tile t); i counts the item's steps
            auto issue_pv = [&](int x, int i, int64_t t) -> bool {
                if (!mbar_wait_short(p_full + x, (np[x] + i) & 1, abort, WT_P)) return false;
                tc_fence_after();
                const uint32_t vbase = opaque_u32(aV + (uint32_t)(t % ST) * C::TILE);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = sdesc_sw128(vbase + kk * 2048, C::BOX, 1024);
                    mma_ts(T_O[x], T_S[x] + kk * 8, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
                }
                return true;
            };
            auto kready = [&](int64_t t) {
                return mbar_wait_short(k_full + t % ST, (uint32_t)(t / ST) & 1, abort, WT_K);
            };
            auto vready = [&](int64_t t) {
                return mbar_wait_short(v_full + t % ST, (uint32_t)(t / ST) & 1, abort, WT_V);
            };

            while (ok && list.next(a, units, p, s, bh)) {
                const int nB = 2 * p + 2;
                // S_A(0): Q_A and the first key tile loaded, O_A / S_A read by the previous epilogue
                if (!(ok = mbar_wait_short(q_full + 0, it & 1, abort, WT_Q))) break;
                if (it > 0 && !(ok = mbar_wait_short(epi_done + 0, (it - 1) & 1, abort, WT_EPI))) break;
                if (!(ok = kready(g))) break;
                tc_fence_after();
                issue_s(0, g);
                if (!(ok = mbar_wait_short(q_full + 1, it & 1, abort, WT_Q))) break;
                if (it > 0 && !(ok = mbar_wait_short(epi_done + 1, (it - 1) & 1, abort, WT_EPI))) break;
                tc_fence_after();
                issue_s(1, g);
                for (int j = 1; ok && j < nB; ++j) {
                    const int64_t tp = g + j - 1, tj = g + j;
                    if (!(ok = vready(tp))) break;
                    if (!(ok = issue_pv(0, j - 1, tp))) break;
                    if (!(ok = kready(tj))) break;
                    tc_fence_after();
                    if (j < nB - 1) issue_s(0, tj);
                    if (!(ok = issue_pv(1, j - 1, tp))) break;
                    mma_commit(kv_empty + tp % ST);
                    issue_s(1, tj);
                }
                if (!ok) break;
                const int64_t tl = g + nB - 1;
                if (!(ok = vready(tl))) break;
                if (!(ok = issue_pv(1, nB - 1, tl))) break;
                mma_commit(kv_empty + tl % ST);
                if (!(ok = mbar_wait_short(m_full, it & 1, abort, WT_M))) break;
                for (int x = 0; ok && x < 2; ++x) {
                    if (!(ok = mbar_wait_short(sq_full + x, it & 1, abort, WT_SQ))) break;
                    tc_fence_after();
                    const uint32_t qbase = opaque_u32(aQ[x]), mbase = opaque_u32(aM);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(T_S[x], sdesc_sw128(qbase + off, 16, 1024),
                               sdesc_sw128(mbase + kk * 2048, C::MBOX, 1024), idO, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(r_full + x);
                }
                np[0] += nB - 1;
                np[1] += nB;
                g += nB;
                ++it;
            }
            mma_commit(mma_done);
            segp_drain(mma_done, 0);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_HIGH));
        // ---------------------------------------------------------------- softmax / epilogue
        const int x = warp >> 2;                          // 0: tile A, 1: tile B
        const int r = threadIdx.x & 127;                  // query row within the tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
        const uint64_t one2 = f2_pack(1.f, 1.f);
        const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
        uint32_t ns = 0;                                  // S phases consumed so far
        int it = 0;
        bool ok = true;
        while (ok && list.next(a, units, p, s, bh)) {
            const int qt = 2 * p + x;                     // q tile index inside the segment
            const int nX = 2 * p + 1 + x;                 // key tiles this tile reads
            float m_used = -INFINITY, l = 0.f;
            for (int i = 0; i < nX; ++i) {
                if (!(ok = mbar_wait(s_full + x, (ns + i) & 1, abort, WT_S))) break;
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
                // P = exp2((S - m) * scale) in bf16, written over the S tile's first 64 columns;
                // scale-and-shift and the partial row sums on packed fp32 pairs
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
            if (!ok) break;
            // sigma(Q_X) over this row, written over Q_X: every Q_X K^T of the item has
            // completed (its last S was read above).  The q_full and m_full waits make the
            // TMA-written Q and z_{s-1} visible to this thread.
            if (!(ok = mbar_wait(q_full + x, it & 1, abort, WT_Q))) break;
            if (!(ok = mbar_wait(m_full, it & 1, abort, WT_M))) break;
            const float den = segp_sigma_row<0, D, D / 8>(sQ[x], r, sZ);
            fence_proxy_async_smem();
            mbar_arrive(sq_full + x);
            if (!(ok = mbar_wait(r_full + x, it & 1, abort, WT_R))) break;
            tc_fence_after();
            const float gt = 1.f / (1.f + __expf(-a.beta[bh % a.H]));
            const float wl = (1.f - gt) / l;
            const float wm = den == 0.f ? 0.f : gt / den;
            // the output row goes to the staging buffer in the layout of a Q tile (128-byte
            // swizzle, 64-column boxes), which is the layout the TMA store reads
            uint8_t *stage = x == 0 ? sQ[0] : (C::B_OUT_IN_M ? sM : sQ[1]);
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
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int ch = ((c & 63) >> 3) + e;
                    *reinterpret_cast<uint4 *>(stage + (c >> 6) * C::BOX + r * 128 + ((ch ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            // O_X and S_X (R_X) have been read: the next item may overwrite them
            tc_fence_before();
            mbar_arrive(epi_done + x);
            fence_proxy_async_smem();
            mbar_arrive(st_ready + x);
            if (r == 0) {
                // one thread stores the tile once every row is staged (rows past L are not
                // written: the store clips at the tensor's extent), waits until the store has
                // read shared memory and releases the buffer to the producer
                if (!(ok = mbar_wait(st_ready + x, it & 1, abort, WT_STAGED))) break;
                const int row0 = s * a.N + qt * 128;
                if (row0 < a.L) {
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_store_3d(&tmO, stage + cb * C::BOX, cb * 64, row0, (int)bh);
                    bulk_commit();
                    bulk_wait_read_all();
                }
                mbar_arrive(out_free + x);
            }
            ns += nX;
            ++it;
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
