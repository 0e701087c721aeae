// Fused Infini-attention forward for 64-token segments and the additive memory rule over
// long sequences: one persistent launch that walks every head in pieces (sm_100a).
//
// The additive update (AI Wiki "Infini-Attention", "How does the compressive memory
// work?") makes the memory before a unit a prefix sum of sigma(K)^T [V | 1] increments
// ("What is linear attention and the delta rule?").  A unit is two segments (128 tokens);
// a piece is up to 16 consecutive units of one head.  For each piece a CTA
//   A. sums the piece's increments on the tensor cores (keys and values read once from
//      HBM), publishes that aggregate and finds the memory before the piece with a
//      decoupled look-back over earlier pieces of the head (Merrill and Garland,
//      "Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016);
//   B. walks the piece's units in order (keys and values now come from L2), carrying the
//      memory in a TMEM accumulator: per unit the local causal softmax of each segment
//      ("What happens inside the Infini-attention block?"), the retrieval
//      sigma(Q) M / sigma(Q) z from the memory before that segment, and the gate.
// The gate is folded into the operands so that one accumulator holds the output: the
// softmax weights are stored already multiplied by (1 - g) / l, and sigma(Q) rows by
// g / (sigma(q) . z), so P V + sigma(Q) M is the gated output (a zero denominator gives a
// zero row, i.e. no memory term).
//
// Warp roles (416 threads): warps 0-1 own the memory rows (TMEM readout, look-back,
// published states); warp 2 issues TMA loads and takes piece tickets; warp 3 issues the
// memory-increment MMAs; warps 4-7 and 8-11 are two work groups that alternate units
// (sigma(K), sigma(Q), softmax, epilogue); warp 12 issues the attention MMAs.
// Pieces are taken by ticket in start order, so a CTA only looks back at pieces taken
// before its own, by CTAs that are running: no wait can depend on a CTA that has not
// started.  Every wait is bounded.
// Layout limits: bf16, d = 64, N = 64, L % 128 == 0.  With several query heads per key/value
// head each query head is a chain of its own (its own pieces, flags and published states);
// keys, values, M0 and z0 are read through the head's key/value head, and the first query
// head of a group writes M_out and z_out.
#pragma once

#include "tc_common.cuh"
#include "tc_small.cuh"

namespace infini {
namespace tc {

struct PieceCfg {
    static constexpr int D = 64, TOK = 128, SEG = 64, ST = 2;
    static constexpr int THREADS = 416;
    static constexpr int MAX_UNITS = 16;              // units per piece
    static constexpr int PREFETCH = 6;                // steps the L2 prefetch runs ahead
    static constexpr int BOX = 128 * 128;             // 128 rows x 64 bf16
    static constexpr int STAGE = 3 * BOX;             // Q, K, V of one unit
    static constexpr int OFF_SK = ST * STAGE;         // sigma(K), one per work group
    // scaled sigma(Q), one per work group: rows 0-63, 64 zero rows, rows 64-127, so the
    // 128-row windows at 0 and at 64 rows are the two segments' rows with zeros elsewhere
    static constexpr int SQB = 3 * 64 * 128;
    static constexpr int OFF_SQ = OFF_SK + 2 * BOX;
    static constexpr int MB = 64 * 128;               // 64 key features x 64 bf16 values
    static constexpr int OFF_M = OFF_SQ + 2 * SQB;    // per group: M before segment 0, 1
    static constexpr int OFF_ONES = OFF_M + 4 * MB;   // [16][128] K-major, row 0 = 1
    static constexpr int ONES = 16 * 128 * 2;
    static constexpr int OFF_Z = OFF_ONES + ONES;     // per group: z before segment 0, 1
    static constexpr int OFF_BAR = OFF_Z + 2 * 2 * 64 * 4;
    static constexpr int NBAR = 32;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr int ROW = 68;                    // published state row: 64 M, z, pad
    static constexpr int STATE = 64 * ROW;
    // TMEM columns: per work group S / P (128) and the output accumulator (64); the
    // memory accumulator (64 values and the z column, 80 with padding) after them
    static constexpr uint32_t T_ACC = 384;
    // threads that read each piece ticket: the two MMA issuers, both work groups, the
    // memory-row warps
    static constexpr int INFO_READERS = 2 + 2 * 128 + 64;
};

__device__ __forceinline__ uint32_t piece_ts(int w) { return (uint32_t)w * 192u; }
__device__ __forceinline__ uint32_t piece_to(int w) { return 128u + (uint32_t)w * 192u; }

struct PieceArgs {
    const float *beta;
    const float *M0, *z0;          // may be NULL
    __nv_bfloat16 *out;
    float *M_out, *z_out;
    int *ticket;                   // zeroed before the launch
    int *flags;                    // [total], zeroed before the launch
    float *agg, *incl;             // [total, 64, ROW]
    int64_t L;
    int U;                         // units per head
    int UP;                        // units per piece (last piece of a head may be shorter)
    int P;                         // pieces per head
    int H, Hkv;
    int chains;                    // query heads (B * H)
    int total;                     // chains * P
};

enum : int { WP_INFO = 601, WP_FULL = 602, WP_KVE = 603, WP_SIG = 604, WP_SKE = 605,
             WP_S = 606, WP_P = 607, WP_PV = 608, WP_O = 609, WP_SQ = 610, WP_M = 611,
             WP_EPI = 612, WP_ACCF = 613, WP_ACCE = 614, WP_LOOK = 615, WP_DRAIN = 616 };

__device__ __forceinline__ void piece_drain(uint64_t *bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > spin_limit()) {
            atomicCAS(&g_wait_status, 0, WP_DRAIN);
            return;
        }
    }
}

__device__ __forceinline__ void tmem_st32_p(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// ex += row r of a published state (64 memory values, then z)
__device__ __forceinline__ void piece_sum(float (&ex)[65], const float *state, int r, bool assign)
{
    const float4 *src = reinterpret_cast<const float4 *>(state + r * PieceCfg::ROW);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float4 x = __ldcg(src + q);
        if (assign) {
            ex[4 * q] = x.x; ex[4 * q + 1] = x.y; ex[4 * q + 2] = x.z; ex[4 * q + 3] = x.w;
        } else {
            ex[4 * q] += x.x; ex[4 * q + 1] += x.y; ex[4 * q + 2] += x.z; ex[4 * q + 3] += x.w;
        }
    }
    const float z = __ldcg(state + r * PieceCfg::ROW + 64);
    ex[64] = assign ? z : ex[64] + z;
}

__device__ __forceinline__ void tmem_st16_zero(uint32_t taddr)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(0u)
        : "memory");
}

__global__ void __launch_bounds__(416, 1)
k_small_pieces(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const PieceArgs a)
{
    using C = PieceCfg;
    constexpr int D = C::D;
    if (__syncthreads_or(threadIdx.x == 0 && wait_status_set())) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    // per load stage w: fullA (keys and values of an A-step), fullB (queries, keys, values
    // of a B-step), kv_empty; per work group / TMEM slot w: the rest
    uint64_t *fullA = bars, *fullB = bars + 2, *kv_empty = bars + 4, *sig_full = bars + 6;
    uint64_t *sk_empty = bars + 8, *s_full = bars + 10, *p_full = bars + 12, *pv_done = bars + 14;
    uint64_t *o_full = bars + 16, *sq_ready = bars + 18, *m_ready = bars + 20, *epi_done = bars + 22;
    uint64_t *acc_full = bars + 24, *acc_free = bars + 25;
    uint64_t *info_full = bars + 26, *info_empty = bars + 28;
    uint64_t *drain_main = bars + 30, *drain_carry = bars + 31;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    volatile int *info = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);      // [2]
    volatile uint32_t *look = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC + 16);   // [6]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(fullA + s, 1);
            mbar_init(fullB + s, 1);
            mbar_init(kv_empty + s, 2);          // carry MMAs and attention MMAs
            mbar_init(sig_full + s, 128);
            mbar_init(sk_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(p_full + s, 128);
            mbar_init(pv_done + s, 1);
            mbar_init(o_full + s, 1);
            mbar_init(sq_ready + s, 128);
            mbar_init(m_ready + s, 64);
            mbar_init(epi_done + s, 128);
            mbar_init(info_full + s, 1);
            mbar_init(info_empty + s, C::INFO_READERS);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_free, 64);
        mbar_init(drain_main, 1);
        mbar_init(drain_carry, 1);
        *abort = 0;
        fence_barrier_init();
    }
    // constants: the ones row of the z column, and the zero rows between the two segments'
    // scaled sigma(Q) rows
    for (int i = threadIdx.x; i < C::ONES / 16; i += blockDim.x) {
        const int row = i / 8;                       // 8 chunks of 16 B per 128-byte row
        const uint32_t one = (row % 16 == 0) ? 0x3F803F80u : 0u;
        *reinterpret_cast<uint4 *>(smem + C::OFF_ONES + i * 16) = make_uint4(one, one, one, one);
    }
    for (int i = threadIdx.x; i < 2 * 64 * 8; i += blockDim.x) {
        const int g = i / (64 * 8), rem = i % (64 * 8);
        *reinterpret_cast<uint4 *>(smem + C::OFF_SQ + g * C::SQB + 64 * 128 + rem * 16) =
            make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (warp == 2) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    auto stage_q = [&](int st) { return smem + st * C::STAGE; };
    auto stage_k = [&](int st) { return smem + st * C::STAGE + C::BOX; };
    auto stage_v = [&](int st) { return smem + st * C::STAGE + 2 * C::BOX; };
    auto sSK = [&](int w) { return smem + C::OFF_SK + w * C::BOX; };
    auto sSQ = [&](int w) { return smem + C::OFF_SQ + w * C::SQB; };
    auto sM = [&](int w, int seg) { return smem + C::OFF_M + (2 * w + seg) * C::MB; };
    float *sZ = reinterpret_cast<float *>(smem + C::OFF_Z);     // [group][seg][64]

    // Every role walks the same sequence of pieces (from the info ring) and, per piece, n
    // A-steps then n B-steps, counting steps g from the start of the CTA.  Step g uses load
    // stage w = g & 1 and belongs to work group w; a B-step also uses TMEM slot w.  So every
    // waiter sees every phase of the barriers it waits on (a parity wait never skips one).
    auto take_info = [&](int k, int &t) -> bool {
        if (!mbar_wait(info_full + (k & 1), (k >> 1) & 1, abort, WP_INFO)) return false;
        t = info[k & 1];
        mbar_arrive(info_empty + (k & 1));
        return true;
    };
    auto piece_units = [&](int t, int &chain, int &pc, int &u0, int &n) {
        chain = t % a.chains;
        pc = t / a.chains;
        u0 = pc * a.UP;
        n = min(a.UP, a.U - u0);
    };

    if (warp == 2) {
        if (lane == 0) {
            // ------------------------------------------------ tickets and TMA producer
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const uint64_t pol_last = l2_policy_evict_last(), pol_first = l2_policy_evict_first();
            // per stage: A- and B-loads issued so far, and the barrier / parity of the last one
            uint32_t g = 0, cA0 = 0, cA1 = 0, cB0 = 0, cB1 = 0, last0 = 0, last1 = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                if (k >= 2 && !(ok = mbar_wait_short(info_empty + (k & 1), ((k >> 1) - 1) & 1, abort, WP_INFO)))
                    break;
                int t = atomicAdd(a.ticket, 1);
                if (t >= a.total) t = -1;
                info[k & 1] = t;
                mbar_arrive(info_full + (k & 1));
                if (t < 0) break;
                int chain, pc, u0, n;
                piece_units(t, chain, pc, u0, n);
                const int kvc = (int)kv_chain(chain, a.H, a.Hkv);
                // L2 prefetch of the piece's tiles a few steps ahead of the loads (the loads
                // are limited to two stages in flight, too few to cover HBM latency alone)
                auto prefetch = [&](int x) {
                    if (x >= 2 * n) return;
                    const int row = (u0 + (x < n ? x : x - n)) * C::TOK;
                    if (x >= n) tma_prefetch_l2_3d(&tmQ, 0, row, chain);
                    tma_prefetch_l2_3d(&tmK, 0, row, kvc);
                    tma_prefetch_l2_3d(&tmV, 0, row, kvc);
                };
                for (int x = 0; x < C::PREFETCH; ++x) prefetch(x);
                for (int phase = 0; ok && phase < 2; ++phase)
                    for (int i = 0; i < n; ++i, ++g) {
                        const int w = g & 1;
                        prefetch(phase * n + i + C::PREFETCH);
                        if (g >= 2 && !(ok = mbar_wait_short(kv_empty + w, ((g >> 1) - 1) & 1, abort, WP_KVE)))
                            break;
                        const int row = (u0 + i) * C::TOK;
                        uint64_t *bar = phase ? fullB + w : fullA + w;
                        const uint32_t use = phase ? (w ? cB1++ : cB0++) : (w ? cA1++ : cA0++);
                        // bits: parity, B (1) or A (0), valid
                        (w ? last1 : last0) = (use & 1) | (phase << 1) | 4;
                        mbar_arrive_expect_tx(bar, (phase ? 3 : 2) * C::BOX);
                        // keys and values stay in L2 from the A-step to the B-step of their
                        // unit; queries and the B-step's second read are last uses
                        const uint64_t pol = phase ? pol_first : pol_last;
                        if (phase) tma_load_3d_hint(stage_q(w), &tmQ, bar, 0, row, chain, pol);
                        tma_load_3d_hint(stage_k(w), &tmK, bar, 0, row, kvc, pol);
                        tma_load_3d_hint(stage_v(w), &tmV, bar, 0, row, kvc, pol);
                    }
            }
            // nothing may still be landing in shared memory when the CTA exits
            if (last0) piece_drain(((last0 >> 1) & 1) ? fullB : fullA, last0 & 1);
            if (last1) piece_drain(((last1 >> 1) & 1) ? fullB + 1 : fullA + 1, last1 & 1);
        }
    } else if (warp == 3) {
        if (lane == 0) {
            // ------------------------------------------------ memory-increment MMAs
            constexpr uint32_t idV = idesc_bf16(128, 64, 1, 1);     // sigma(K)^T V
            constexpr uint32_t idZ = idesc_bf16(128, 16, 1, 0);     // sigma(K)^T 1
            const uint32_t aOnes = smem_u32(smem + C::OFF_ONES);
            uint32_t g = 0, cA0 = 0, cA1 = 0, cB0 = 0, cB1 = 0, nfree = 0;
            bool ok = true, first = true;
            // rows 64-127 of the A operand (features 64-127 do not exist) read whatever
            // follows sigma(K) in shared memory; those TMEM lanes are never read
            auto incr = [&](uint32_t aSK, uint32_t aV, int k0, int k1, bool fresh) {
                for (int kk = k0; kk < k1; ++kk) {
                    const uint64_t da = sdesc_sw128(aSK + kk * 2048, C::BOX, 1024);
                    const uint32_t acc = (fresh && kk == k0) ? 0u : 1u;
                    mma_ss(tmem + C::T_ACC, da, sdesc_sw128(aV + kk * 2048, C::BOX, 1024), idV, acc);
                    mma_ss(tmem + C::T_ACC + 64, da,
                           sdesc_sw128(aOnes + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024), idZ, acc);
                }
            };
            auto wait_free = [&]() -> bool {
                const bool r = mbar_wait_short(acc_free, nfree & 1, abort, WP_ACCE);
                ++nfree;
                return r;
            };
            for (int k = 0; ok; ++k) {
                int t;
                if (!(ok = take_info(k, t)) || t < 0) break;
                int chain, pc, u0, n;
                piece_units(t, chain, pc, u0, n);
                for (int i = 0; ok && i < n; ++i, ++g) {                 // A-steps
                    const int w = g & 1;
                    if (!(ok = mbar_wait_short(fullA + w, (w ? cA1++ : cA0++) & 1, abort, WP_FULL))) break;
                    if (!(ok = mbar_wait_short(sig_full + w, (g >> 1) & 1, abort, WP_SIG))) break;
                    if (i == 0 && !first && !(ok = wait_free())) break;
                    first = false;
                    tc_fence_after();
                    incr(smem_u32(sSK(w)), smem_u32(stage_v(w)), 0, 8, i == 0);
                    mma_commit(sk_empty + w);
                    mma_commit(kv_empty + w);
                    mma_commit(kv_empty + w);
                    if (i == n - 1) mma_commit(acc_full);
                }
                for (int i = 0; ok && i < n; ++i, ++g) {                 // B-steps
                    const int w = g & 1;
                    if (!(ok = mbar_wait_short(fullB + w, (w ? cB1++ : cB0++) & 1, abort, WP_FULL))) break;
                    if (!(ok = mbar_wait_short(sig_full + w, (g >> 1) & 1, abort, WP_SIG))) break;
                    if (!(ok = wait_free())) break;                          // memory before the unit
                    tc_fence_after();
                    incr(smem_u32(sSK(w)), smem_u32(stage_v(w)), 0, 4, false);
                    mma_commit(acc_full);
                    if (!(ok = wait_free())) break;                          // before its 2nd segment
                    tc_fence_after();
                    incr(smem_u32(sSK(w)), smem_u32(stage_v(w)), 4, 8, false);
                    mma_commit(acc_full);
                    mma_commit(sk_empty + w);
                    mma_commit(kv_empty + w);
                }
            }
            mma_commit(drain_carry);
            piece_drain(drain_carry, 0);
        }
    } else if (warp == 12) {
        if (lane == 0) {
            // ------------------------------------------------ attention MMAs
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idO = idesc_bf16(128, 64, 0, 1);
            uint32_t g = 0, cB0 = 0, cB1 = 0;
            bool ok = true, have_prev = false;
            int pw = 0, pj = 0;
            // P V of a unit, then its retrieval added to the same accumulator
            auto finish = [&](int y, int jy) -> bool {
                if (!mbar_wait_short(p_full + y, jy & 1, abort, WP_P)) return false;
                if (jy >= 1 && !mbar_wait_short(epi_done + y, (jy - 1) & 1, abort, WP_EPI)) return false;
                tc_fence_after();
                const uint32_t aV = smem_u32(stage_v(y));
                for (int kk = 0; kk < C::TOK / 16; ++kk)
                    mma_ts(tmem + piece_to(y), tmem + piece_ts(y) + kk * 8,
                           sdesc_sw128(aV + kk * 2048, C::BOX, 1024), idO, kk > 0 ? 1u : 0u);
                mma_commit(pv_done + y);
                mma_commit(kv_empty + y);
                if (!mbar_wait_short(sq_ready + y, jy & 1, abort, WP_SQ)) return false;
                if (!mbar_wait_short(m_ready + y, jy & 1, abort, WP_M)) return false;
                tc_fence_after();
                const uint32_t aSQ = smem_u32(sSQ(y));
                const uint32_t aM0 = smem_u32(sM(y, 0)), aM1 = smem_u32(sM(y, 1));
                for (int kk = 0; kk < D / 16; ++kk) {
                    mma_ss(tmem + piece_to(y), sdesc_sw128(aSQ + kk * 32, 16, 1024),
                           sdesc_sw128(aM0 + kk * 2048, C::MB, 1024), idO, 1u);
                    mma_ss(tmem + piece_to(y), sdesc_sw128(aSQ + 64 * 128 + kk * 32, 16, 1024),
                           sdesc_sw128(aM1 + kk * 2048, C::MB, 1024), idO, 1u);
                }
                mma_commit(o_full + y);
                return true;
            };
            for (int k = 0; ok; ++k) {
                int t;
                if (!(ok = take_info(k, t)) || t < 0) break;
                int chain, pc, u0, n;
                piece_units(t, chain, pc, u0, n);
                // finish the last unit of the previous piece now: its stage must be free
                // before the producer can load this piece's A-steps and first B-step
                if (have_prev && !(ok = finish(pw, pj))) break;
                have_prev = false;
                g += n;                                                     // A-steps
                for (int i = 0; ok && i < n; ++i, ++g) {                   // B-steps
                    const int w = g & 1, j = w ? cB1++ : cB0++;
                    if (!(ok = mbar_wait_short(fullB + w, j & 1, abort, WP_FULL))) break;
                    if (j >= 1 && !(ok = mbar_wait_short(pv_done + w, (j - 1) & 1, abort, WP_PV))) break;
                    tc_fence_after();
                    const uint32_t aQ = smem_u32(stage_q(w)), aK = smem_u32(stage_k(w));
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + piece_ts(w), sdesc_sw128(aQ + kk * 32, 16, 1024),
                               sdesc_sw128(aK + kk * 32, 16, 1024), idS, kk > 0 ? 1u : 0u);
                    mma_commit(s_full + w);
                    if (have_prev && !(ok = finish(pw, pj))) break;
                    have_prev = true;
                    pw = w;
                    pj = j;
                }
            }
            if (ok && have_prev) finish(pw, pj);
            mma_commit(drain_main);
            piece_drain(drain_main, 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------- work groups (one row each)
        const int wg = (warp - 4) >> 2;
        const int r = threadIdx.x - 128 - wg * 128;              // token of the unit
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int rr = r < 64 ? r : r + 64;                      // row in the sigma(Q) buffer
        uint32_t g = 0, cA = 0, cB = 0;                          // this group's A- / B-steps
        bool ok = true;
        // sigma of row r of a 128 x 64 tile into row dr of dst (same swizzle: dr % 8 == r % 8),
        // as elu1 on packed fp32 pairs.  Two chunks per iteration: fully unrolled, with five
        // roles on each SM sub-partition, instruction-cache misses cost more than the loop.
        const uint64_t one2 = f2_pack(1.f, 1.f);
        const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
        auto sigma_row_to = [&](const uint8_t *src, uint8_t *dst, int dr) {
#pragma unroll 2
            for (int ch = 0; ch < 8; ++ch) {
                const int c = (ch ^ (r & 7)) << 4;
                const uint4 x = *reinterpret_cast<const uint4 *>(src + r * 128 + c);
                uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = __uint_as_float(w4[e] << 16), x1 = __uint_as_float(w4[e] & 0xffff0000u);
                    float a0, a1, p0, p1;
                    f2_unpack(f2_mul(f2_pack(fminf(x0, 0.f), fminf(x1, 0.f)), log2e2), a0, a1);
                    f2_unpack(f2_add(f2_pack(x0, x1), one2), p0, p1);
                    w4[e] = pack_bf16x2(fmaxf(p0, ex2(a0)), fmaxf(p1, ex2(a1)));
                }
                *reinterpret_cast<uint4 *>(dst + dr * 128 + c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        };
        // sigma(K) of this group's step g into its buffer, once the carry has used the last one
        auto sigma_k = [&]() -> bool {
            const uint32_t uses = g >> 1;                        // earlier steps of this group
            if (uses >= 1 && !mbar_wait(sk_empty + wg, (uses - 1) & 1, abort, WP_SKE)) return false;
            sigma_row_to(stage_k(wg), sSK(wg), r);
            fence_proxy_async_smem();
            mbar_arrive(sig_full + wg);
            return true;
        };
        const float kscale = rsqrtf((float)D) * 1.4426950408889634f;
        for (int k = 0; ok; ++k) {
            int t;
            if (!(ok = take_info(k, t)) || t < 0) break;
            int chain, pc, u0, n;
            piece_units(t, chain, pc, u0, n);
            const float gate = 1.f / (1.f + __expf(-a.beta[chain % a.H]));
            for (int i = 0; ok && i < n; ++i, ++g) {                     // A-steps
                if ((int)(g & 1) != wg) continue;
                if (!(ok = mbar_wait(fullA + wg, cA++ & 1, abort, WP_FULL))) break;
                ok = sigma_k();
            }
            for (int i = 0; ok && i < n; ++i, ++g) {                     // B-steps
                if ((int)(g & 1) != wg) continue;
                const uint32_t j = cB++;
                if (!(ok = mbar_wait(fullB + wg, j & 1, abort, WP_FULL))) break;
                if (!(ok = sigma_k())) break;
                // sigma(Q) of row r into its row of the group's buffer; scaled once z is known
                // (the buffer is free: this group's previous retrieval ran before its epilogue)
                sigma_row_to(stage_q(wg), sSQ(wg), rr);
                // local softmax of row r over its own segment's keys, weights times (1-g)/l
                if (!(ok = mbar_wait(s_full + wg, j & 1, abort, WP_S))) break;
                tc_fence_after();
                {
                    const int lo = (r >> 6) << 6;
                    const uint32_t tS = tmem + piece_ts(wg);
                    uint32_t v[2][32];
                    tmem_ld32(lane_base + tS + lo, v[0]);
                    tmem_ld32(lane_base + tS + lo + 32, v[1]);
                    tmem_ld_wait();
                    float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (lo + c * 32 + e > r) v[c][e] = __float_as_uint(-INFINITY);
                            pm[e & 3] = fmaxf(pm[e & 3], __uint_as_float(v[c][e]));
                        }
                    const float mk = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) * kscale;
                    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float p = ex2(fmaf(__uint_as_float(v[c][e]), kscale, -mk));
                            ps[e & 3] += p;
                            v[c][e] = __float_as_uint(p);
                        }
                    const float wl = (1.f - gate) / ((ps[0] + ps[1]) + (ps[2] + ps[3]));
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(v[c][2 * e]) * wl,
                                                __uint_as_float(v[c][2 * e + 1]) * wl);
                        tmem_st16_s(lane_base + tS + (lo >> 1) + c * 16, pk);
                        tmem_st16_zero(lane_base + tS + ((64 - lo) >> 1) + c * 16);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(p_full + wg);
                }
                // sigma(Q) scaled by g / (sigma(q) . z) with z before this row's segment
                if (!(ok = mbar_wait(m_ready + wg, j & 1, abort, WP_M))) break;
                {
                    const float *zz = sZ + (wg * 2 + (r >> 6)) * 64;
                    uint8_t *row = sSQ(wg) + rr * 128;
                    uint4 q4[8];
                    uint64_t dp2[2] = {0ull, 0ull};
                    const float2 *z2 = reinterpret_cast<const float2 *>(zz);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        q4[ch] = *reinterpret_cast<const uint4 *>(row + ((ch ^ (rr & 7)) << 4));
                        const uint32_t w4[4] = {q4[ch].x, q4[ch].y, q4[ch].z, q4[ch].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 zp = z2[ch * 4 + e];
                            dp2[e & 1] = f2_fma(f2_pack(__uint_as_float(w4[e] << 16), __uint_as_float(w4[e] & 0xffff0000u)),
                                                f2_pack(zp.x, zp.y), dp2[e & 1]);
                        }
                    }
                    float d0, d1, d2, d3;
                    f2_unpack(dp2[0], d0, d1);
                    f2_unpack(dp2[1], d2, d3);
                    const float den = (d0 + d1) + (d2 + d3);
                    const float wm = den == 0.f ? 0.f : gate / den;
                    const uint64_t wm2 = f2_pack(wm, wm);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t w4[4] = {q4[ch].x, q4[ch].y, q4[ch].z, q4[ch].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float y0, y1;
                            f2_unpack(f2_mul(f2_pack(__uint_as_float(w4[e] << 16), __uint_as_float(w4[e] & 0xffff0000u)), wm2),
                                      y0, y1);
                            w4[e] = pack_bf16x2(y0, y1);
                        }
                        *reinterpret_cast<uint4 *>(row + ((ch ^ (rr & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(sq_ready + wg);
                }
                // epilogue: the accumulator already holds the gated output row
                if (!(ok = mbar_wait(o_full + wg, j & 1, abort, WP_O))) break;
                tc_fence_after();
                {
                    __nv_bfloat16 *orow = a.out + (chain * a.L + (int64_t)(u0 + i) * C::TOK + r) * D;
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + tmem + piece_to(wg) + c, o);
                        tmem_ld_wait();
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)   // streaming: the output is not read again
                            __stcs(dst + e, make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]));
                    }
                    tc_fence_before();
                    mbar_arrive(epi_done + wg);
                }
            }
        }
    } else {
        // ---------------------------------------------------- memory rows (warps 0-1)
        const int r = threadIdx.x;                               // key feature 0..63
        const uint32_t tACC = tmem + C::T_ACC + ((uint32_t)(warp * 32) << 16);
        uint32_t g = 0, cB0 = 0, cB1 = 0, nfull = 0;            // steps; B-steps per slot
        bool ok = true;
        float ex[D + 1];                                         // memory before the piece
        auto wait_full = [&]() -> bool {
            const bool res = mbar_wait(acc_full, nfull & 1, abort, WP_ACCF);
            ++nfull;
            if (res) tc_fence_after();
            return res;
        };
        // the accumulator's row as a bf16 B operand (key feature r, 64 values) and z as fp32
        auto mem_from_acc = [&](int grp, int seg) {
            uint8_t *dst = sM(grp, seg);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t x[32];
                tmem_ld32(tACC + h * 32, x);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int ch = h * 4 + c;
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w4[e] = pack_bf16x2(__uint_as_float(x[8 * c + 2 * e]), __uint_as_float(x[8 * c + 2 * e + 1]));
                    *reinterpret_cast<uint4 *>(dst + r * 128 + ((ch ^ (r & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            uint32_t zc[16];
            tmem_ld16(tACC + 64, zc);
            tmem_ld_wait();
            sZ[(grp * 2 + seg) * 64 + r] = __uint_as_float(zc[0]);
        };
        // a slot's memory buffers are free once its previous unit's retrieval has run
        auto wait_slot = [&](int w) -> bool {
            const uint32_t c = w ? cB1 : cB0;
            return c == 0 || mbar_wait(o_full + w, (c - 1) & 1, abort, WP_O);
        };
        for (int k = 0; ok; ++k) {
            int t;
            if (!(ok = take_info(k, t)) || t < 0) break;
            int chain, pc, u0, n;
            piece_units(t, chain, pc, u0, n);
            const bool last = pc == a.P - 1;
            const int64_t kvc = kv_chain(chain, a.H, a.Hkv);
            const bool state_writer = (chain % a.H) % (a.H / a.Hkv) == 0;   // first query head of its group
            g += n;                                                   // A-steps
            // ---- the piece's aggregate, published for later pieces of the head
            if (!(ok = wait_full())) break;
            if (pc > 0) {
                float4 *dst = reinterpret_cast<float4 *>(a.agg + (int64_t)t * C::STATE + r * C::ROW);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t x[32];
                    tmem_ld32(tACC + h * 32, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[h * 8 + q] = make_float4(__uint_as_float(x[4 * q]), __uint_as_float(x[4 * q + 1]),
                                                     __uint_as_float(x[4 * q + 2]), __uint_as_float(x[4 * q + 3]));
                }
                uint32_t zc[16];
                tmem_ld16(tACC + 64, zc);
                tmem_ld_wait();
                dst[D / 4] = make_float4(__uint_as_float(zc[0]), 0.f, 0.f, 0.f);
            }
            __threadfence();
            asm volatile("bar.sync 1, 64;" ::: "memory");
            if (r == 0 && pc > 0) st_release_gpu(a.flags + t, FLAG_AGG);
            // ---- look-back: the memory before the piece
            if (pc == 0) {
#pragma unroll
                for (int e = 0; e <= D; ++e) ex[e] = 0.f;
                if (a.M0) {
                    const float4 *m = reinterpret_cast<const float4 *>(a.M0 + (kvc * D + r) * D);
#pragma unroll
                    for (int q = 0; q < D / 4; ++q) {
                        const float4 x = m[q];
                        ex[4 * q] = x.x; ex[4 * q + 1] = x.y; ex[4 * q + 2] = x.z; ex[4 * q + 3] = x.w;
                    }
                }
                if (a.z0) ex[D] = a.z0[kvc * D + r];
            } else {
                // thread i watches predecessor pc-1-i; the walk ends at the nearest piece
                // that has published its inclusive prefix, and every piece after it must
                // have published its aggregate (piece 0 publishes only its inclusive prefix)
                const int pred = pc - 1 - r;
                const long long t0 = clock64();
                int stop = -1;
                while (true) {
                    const int f = pred >= 0 ? ld_acquire_gpu(a.flags + chain + (int64_t)pred * a.chains) : 0;
                    const uint32_t inc = __ballot_sync(0xffffffffu, pred >= 0 && f == FLAG_INCL);
                    const uint32_t none = __ballot_sync(0xffffffffu, pred >= 0 && f == 0);
                    const uint32_t quit = __ballot_sync(0xffffffffu, *abort != 0 || clock64() - t0 > spin_limit());
                    if (lane == 0) {
                        look[warp * 3] = inc;
                        look[warp * 3 + 1] = none;
                        look[warp * 3 + 2] = quit;
                    }
                    asm volatile("bar.sync 1, 64;" ::: "memory");
                    const uint64_t inc64 = (uint64_t)look[0] | ((uint64_t)look[3] << 32);
                    const uint64_t none64 = (uint64_t)look[1] | ((uint64_t)look[4] << 32);
                    const bool give_up = (look[2] | look[5]) != 0;
                    asm volatile("bar.sync 1, 64;" ::: "memory");
                    // every thread of both warps read the same words, so all take the same exit
                    if (inc64 != 0) {
                        const int first = __ffsll((long long)inc64) - 1;
                        const uint64_t before = first == 0 ? 0ull : (none64 & ((1ull << first) - 1));
                        if (before == 0) {
                            stop = first;
                            break;
                        }
                    }
                    if (give_up) {
                        if (r == 0) atomicCAS(&g_wait_status, 0, WP_LOOK);
                        *abort = 1;
                        break;
                    }
                    __nanosleep(64);
                }
                if (stop < 0) {
                    ok = false;
                    break;
                }
                piece_sum(ex, a.incl + ((int64_t)chain + (int64_t)(pc - 1 - stop) * a.chains) * C::STATE, r, true);
                for (int q = stop - 1; q >= 0; --q)
                    piece_sum(ex, a.agg + ((int64_t)chain + (int64_t)(pc - 1 - q) * a.chains) * C::STATE, r, false);
            }
            // ---- inclusive prefix (or the head's final memory): ex plus the aggregate, which
            // the accumulator still holds (the carry waits for this role before reusing it)
            {
                // the head's final memory goes to M_out from the first query head of its group
                // only; the other heads of the group skip it (their incl is never read)
                float *dst = last ? (state_writer ? a.M_out + (kvc * D + r) * D : nullptr)
                                  : a.incl + (int64_t)t * C::STATE + r * C::ROW;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t x[32];
                    tmem_ld32(tACC + h * 32, x);
                    tmem_ld_wait();
                    if (dst)
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const int c = h * 32 + 4 * q;
                            reinterpret_cast<float4 *>(dst)[h * 8 + q] =
                                make_float4(ex[c] + __uint_as_float(x[4 * q]), ex[c + 1] + __uint_as_float(x[4 * q + 1]),
                                            ex[c + 2] + __uint_as_float(x[4 * q + 2]), ex[c + 3] + __uint_as_float(x[4 * q + 3]));
                        }
                }
                uint32_t zc[16];
                tmem_ld16(tACC + 64, zc);
                tmem_ld_wait();
                const float zi = ex[D] + __uint_as_float(zc[0]);
                if (last) {
                    if (state_writer) a.z_out[kvc * D + r] = zi;
                } else {
                    reinterpret_cast<float4 *>(dst)[D / 4] = make_float4(zi, 0.f, 0.f, 0.f);
                }
            }
            __threadfence();
            asm volatile("bar.sync 1, 64;" ::: "memory");
            if (r == 0 && !last) st_release_gpu(a.flags + t, FLAG_INCL);
            // ---- the carry starts from the memory before the piece
            {
                uint32_t x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __float_as_uint(ex[e]);
                tmem_st32_p(tACC, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = __float_as_uint(ex[32 + e]);
                tmem_st32_p(tACC + 32, x);
                uint32_t zc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) zc[e] = 0u;
                zc[0] = __float_as_uint(ex[D]);
                tmem_st16_s(tACC + 64, zc);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(acc_free);
            if (!(ok = wait_slot(g & 1))) break;
            {
                uint8_t *dst = sM(g & 1, 0);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w4[e] = pack_bf16x2(ex[ch * 8 + 2 * e], ex[ch * 8 + 2 * e + 1]);
                    *reinterpret_cast<uint4 *>(dst + r * 128 + ((ch ^ (r & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                sZ[((g & 1) * 2) * 64 + r] = ex[D];
            }
            // ---- the units: memory before each segment, for the retrieval
            for (int i = 0; ok && i < n; ++i, ++g) {
                const int w = g & 1;
                if (!(ok = wait_full())) break;                       // after segment 0
                mem_from_acc(w, 1);
                tc_fence_before();
                mbar_arrive(acc_free);
                fence_proxy_async_smem();
                mbar_arrive(m_ready + w);
                if (w) ++cB1; else ++cB0;
                // the next unit's buffers must be free before its memory is written
                if (i + 1 < n && !(ok = wait_slot(w ^ 1))) break;
                if (!(ok = wait_full())) break;                       // after the unit
                if (i + 1 < n) mem_from_acc(w ^ 1, 0);
                tc_fence_before();
                mbar_arrive(acc_free);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc
}  // namespace infini
