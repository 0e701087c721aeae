// Token-by-token decode of the Infini-attention forward.
//
// A stream produced one token at a time keeps the forward's segments: the token at position
// t of a head belongs to segment s = t / N at offset p = t % N.  Its local attention spans
// the keys of segment s at offsets 0..p, its retrieval reads the memory from before
// segment s, and once offset N - 1 has been processed the whole segment is folded into the
// memory (AI Wiki "Infini-Attention", "What happens inside the Infini-attention block?"
// and "How does the compressive memory work?"; the Hugging Face reproduction,
// "Infini-Attention Mechanism", steps 1-6).  So feeding a sequence through the decode step
// gives the forward's outputs token for token, and after the last fold its memory.
//
// The caller owns the key/value cache of the current segment, [B, Hkv, N, d] in the
// activation dtype, and the memory (M, z) in fp32.  The step writes the new token's key and
// value into cache row p; the fold is a separate launch on the same stream (the state
// kernels of the CUDA-core path, run on the cache as one segment).
#pragma once

#include <cooperative_groups.h>

#include "simt_kernels.cuh"

namespace infini {

namespace cg = cooperative_groups;

// ---------------------------------------------------------------------------------------
// Decode, split over a thread-block cluster.  The cluster's CL CTAs share one (batch, key/
// value head) and all G <= 8 query heads of its group, so each cached key and value is read
// once for the whole group; CTA r takes the r-th slice of the keys 0..pos and walks it in
// tiles of KT keys.  Per tile: every thread issues asynchronous 16-byte copies
// (cp.async) of the tile's key and value rows into shared memory, all in flight at once
// (one memory round trip per tile), thread j forms the G
// scores of key j (padded key rows keep the 16-byte reads conflict-free), warp g updates
// head g's running max and sum, and each thread accumulates its (head, column) outputs
// over the tile's values.  After a cluster barrier CTA 0 reads every CTA's (max, sum,
// weighted values) through distributed shared memory, merges them, adds the retrieval
// sigma(q_g) M / (sigma(q_g) . z) and the gate, and writes the outputs; CTA 0 starts the
// copy of M and z into its shared memory first thing, so it overlaps the attention.  The
// second cluster barrier keeps every CTA's shared memory alive until CTA 0 is done.  The
// CTA whose slice holds key pos writes this token's key and value into cache row pos; the
// tile takes that row from the call's own inputs.
// ---------------------------------------------------------------------------------------
constexpr int kDecodeGMax = 8;

template <typename T, int D>
struct DecCfg {
    static constexpr int E = (int)sizeof(T);
    static constexpr int GM = kDecodeGMax;
    static constexpr int KT = E == 2 ? 256 : 128;        // keys per tile
    static constexpr int KROW = D + 16 / E;              // padded key row, elements
    static constexpr int CPR = D * E / 16;               // 16-byte chunks per row
    static constexpr int OPT = (GM * D + 255) / 256;     // outputs per thread at most
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KT * KROW * E;
    static constexpr int OFF_P = OFF_V + KT * D * E;     // [GM][KT] scores, then weights
    static constexpr int OFF_Q = OFF_P + GM * KT * 4;    // [GM][D] q * scale * log2(e)
    static constexpr int OFF_SQ = OFF_Q + GM * D * 4;    // [GM][D] sigma(q)
    static constexpr int OFF_CO = OFF_SQ + GM * D * 4;   // [GM][D] this CTA's weighted values
    static constexpr int OFF_ST = OFF_CO + GM * D * 4;   // max, sum, rescale, den: [4][GM]
    static constexpr int OFF_MS = OFF_ST + 4 * GM * 4;   // [D][D] M (CTA 0)
    static constexpr int OFF_Z = OFF_MS + D * D * 4;     // [D] z (CTA 0)
    static constexpr int BYTES = OFF_Z + D * 4;
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(smem_dst)),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <typename T>
__device__ __forceinline__ float dot_row(const float *q, const T *k, int n);
template <>
__device__ __forceinline__ float dot_row(const float *q, const __nv_bfloat16 *k, int n)
{
    float s = 0.f;
    for (int c = 0; c < n; c += 8) {
        const uint4 u = *reinterpret_cast<const uint4 *>(k + c);
        const float4 qa = *reinterpret_cast<const float4 *>(q + c);
        const float4 qb = *reinterpret_cast<const float4 *>(q + c + 4);
        s = fmaf(qa.x, __uint_as_float(u.x << 16), s);
        s = fmaf(qa.y, __uint_as_float(u.x & 0xFFFF0000u), s);
        s = fmaf(qa.z, __uint_as_float(u.y << 16), s);
        s = fmaf(qa.w, __uint_as_float(u.y & 0xFFFF0000u), s);
        s = fmaf(qb.x, __uint_as_float(u.z << 16), s);
        s = fmaf(qb.y, __uint_as_float(u.z & 0xFFFF0000u), s);
        s = fmaf(qb.z, __uint_as_float(u.w << 16), s);
        s = fmaf(qb.w, __uint_as_float(u.w & 0xFFFF0000u), s);
    }
    return s;
}
template <>
__device__ __forceinline__ float dot_row(const float *q, const float *k, int n)
{
    float s = 0.f;
    for (int c = 0; c < n; c += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(k + c);
        const float4 qa = *reinterpret_cast<const float4 *>(q + c);
        s = fmaf(qa.x, x.x, s);
        s = fmaf(qa.y, x.y, s);
        s = fmaf(qa.z, x.z, s);
        s = fmaf(qa.w, x.w, s);
    }
    return s;
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
k_decode_split(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
               const float *__restrict__ beta, T *k_cache, T *v_cache, int pos, int N,
               const float *__restrict__ M, const float *__restrict__ z, T *__restrict__ out,
               int H, int Hkv)
{
    using C = DecCfg<T, D>;
    constexpr int GM = C::GM, KT = C::KT, OPT = C::OPT;
    extern __shared__ __align__(16) uint8_t dsm[];
    T *sK = reinterpret_cast<T *>(dsm + C::OFF_K);
    T *sV = reinterpret_cast<T *>(dsm + C::OFF_V);
    float *sP = reinterpret_cast<float *>(dsm + C::OFF_P);
    float *sQ = reinterpret_cast<float *>(dsm + C::OFF_Q);
    float *sSQ = reinterpret_cast<float *>(dsm + C::OFF_SQ);
    float *sCO = reinterpret_cast<float *>(dsm + C::OFF_CO);
    float *sM = reinterpret_cast<float *>(dsm + C::OFF_ST);
    float *sL = sM + GM, *sA = sL + GM, *sDen = sA + GM;
    float *sMem = reinterpret_cast<float *>(dsm + C::OFF_MS);
    float *sZ = reinterpret_cast<float *>(dsm + C::OFF_Z);

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank(), CL = (int)cluster.num_blocks();
    const int64_t chain = blockIdx.x / CL;
    const int G = H / Hkv;
    const int64_t b = chain / Hkv;
    const int kvh = (int)(chain % Hkv);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const T *kt = k + chain * D, *vt = v + chain * D;
    T *Kc = k_cache + chain * (int64_t)N * D, *Vc = v_cache + chain * (int64_t)N * D;
    const int64_t h0 = b * H + (int64_t)kvh * G;      // first query head of the group

    if (rank == 0) {                                   // the memory, for the retrieval
        const float *Mc = M + chain * D * D;
        for (int i = tid; i < D * D / 4; i += 256) cp_async16(sMem + 4 * i, Mc + 4 * i);
        for (int i = tid; i < D / 4; i += 256) cp_async16(sZ + 4 * i, z + chain * D + 4 * i);
        cp_async_commit();
    }
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    for (int i = tid; i < GM * D; i += 256) {
        const float x = i / D < G ? ld_f(q + h0 * D + i) : 0.f;
        sQ[i] = x * sl2;
        sSQ[i] = feature_map(x);
    }
    if (tid < GM) {
        sM[tid] = -INFINITY;
        sL[tid] = 0.f;
    }
    const int total = pos + 1, chunk = (total + CL - 1) / CL;
    const int j0 = rank * chunk, j1 = min(j0 + chunk, total);
    if (j0 <= pos && pos < j1)
        for (int i = tid; i < D; i += 256) {
            Kc[(int64_t)pos * D + i] = kt[i];
            Vc[(int64_t)pos * D + i] = vt[i];
        }
    float o[OPT];
#pragma unroll
    for (int u = 0; u < OPT; ++u) o[u] = 0.f;
    __syncthreads();

    for (int t0 = j0; t0 < j1; t0 += KT) {
        const int nt = min(KT, j1 - t0);
        for (int i = tid; i < nt * C::CPR; i += 256) {
            const int row = i / C::CPR, ch = i % C::CPR, j = t0 + row;
            const T *kr = j == pos ? kt : Kc + (int64_t)j * D;
            const T *vr = j == pos ? vt : Vc + (int64_t)j * D;
            cp_async16(sK + row * C::KROW + ch * (16 / C::E), kr + ch * (16 / C::E));
            cp_async16(sV + row * D + ch * (16 / C::E), vr + ch * (16 / C::E));
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        if (tid < nt)
            for (int g = 0; g < G; ++g) sP[g * KT + tid] = dot_row(sQ + g * D, sK + tid * C::KROW, D);
        __syncthreads();
        if (warp < G) {                                // warp g: head g's max, weights, sum
            float *pg = sP + warp * KT;
            float mx = -INFINITY;
            for (int j = lane; j < nt; j += 32) mx = fmaxf(mx, pg[j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mo = sM[warp], mn = fmaxf(mo, mx);
            float sum = 0.f;
            for (int j = lane; j < nt; j += 32) {
                const float p = exp2f(pg[j] - mn);
                pg[j] = p;
                sum += p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane == 0) {
                const float a = exp2f(mo - mn);        // 0 before the first tile
                sA[warp] = a;
                sL[warp] = sL[warp] * a + sum;
                sM[warp] = mn;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < OPT; ++u) {
            const int i = tid + 256 * u;
            if (i < G * D) {
                const int g = i / D, c = i % D;
                const float *pg = sP + g * KT;
                float acc = o[u] * sA[g];
#pragma unroll 8
                for (int j = 0; j < nt; ++j) acc = fmaf(pg[j], ld_f(sV + j * D + c), acc);
                o[u] = acc;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < OPT; ++u) {
        const int i = tid + 256 * u;
        if (i < G * D) sCO[i] = o[u];
    }
    // CTA 0: the retrieval while the other CTAs finish
    float num[OPT];
    if (rank == 0) {
        cp_async_wait_all();                           // M and z (a CTA without keys)
        __syncthreads();
        if (warp < G) {
            float part = 0.f;
            for (int f = lane; f < D; f += 32) part = fmaf(sSQ[warp * D + f], sZ[f], part);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
            if (lane == 0) sDen[warp] = part;
        }
#pragma unroll
        for (int u = 0; u < OPT; ++u) {
            const int i = tid + 256 * u;
            num[u] = 0.f;
            if (i < G * D) {
                const int g = i / D, c = i % D;
                float acc = 0.f;
#pragma unroll 8
                for (int f = 0; f < D; ++f) acc = fmaf(sSQ[g * D + f], sMem[f * D + c], acc);
                num[u] = acc;
            }
        }
    }
    cluster.sync();
    if (rank == 0) {
#pragma unroll
        for (int u = 0; u < OPT; ++u) {
            const int i = tid + 256 * u;
            if (i >= G * D) continue;
            const int g = i / D;
            float mx = -INFINITY;
            for (int r = 0; r < CL; ++r) mx = fmaxf(mx, *cluster.map_shared_rank(sM + g, r));
            float os = 0.f, ls = 0.f;
            for (int r = 0; r < CL; ++r) {
                const float rm = *cluster.map_shared_rank(sM + g, r);
                if (rm == -INFINITY) continue;       // a CTA without keys
                const float sc = exp2f(rm - mx);
                os = fmaf(*cluster.map_shared_rank(sCO + i, r), sc, os);
                ls = fmaf(*cluster.map_shared_rank(sL + g, r), sc, ls);
            }
            const float den = sDen[g];
            const float amem = den == 0.f ? 0.f : num[u] / den;
            const float gt = 1.f / (1.f + expf(-beta[kvh * G + g]));
            st_f(out + h0 * D + i, gt * amem + (1.f - gt) * (os / ls));
        }
    }
    cluster.sync();
}

// One CTA per (batch, query head).  Eight warps split the keys 0..p; each keeps an online
// softmax (running max, sum and weighted values, d / 32 columns per lane), merged through
// shared memory.  The retrieval sigma(q) M / (sigma(q) . z) and the gate follow.  Row p of
// the cache is written by the group's first query head only, and no CTA reads it: the
// current key and value come from the step's own inputs.
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_decode_attn(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ beta, T *k_cache, T *v_cache, int pos, int N,
              const float *__restrict__ M, const float *__restrict__ z, T *__restrict__ out,
              int H, int Hkv)
{
    constexpr int NW = 8, PL = D / 32, PARTS = 256 / D, FP = D / PARTS;
    __shared__ float s_sq[D];
    __shared__ float s_m[NW], s_l[NW];
    __shared__ float s_o[NW][D];
    __shared__ float s_num[PARTS][D];
    __shared__ float s_den;

    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int G = H / Hkv, kvh = h / G;
    const int64_t chain = b * Hkv + kvh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const T *qt = q + bh * D;
    const T *kt = k + chain * D, *vt = v + chain * D;
    T *Kc = k_cache + chain * (int64_t)N * D, *Vc = v_cache + chain * (int64_t)N * D;

    for (int i = tid; i < D; i += 256) s_sq[i] = feature_map(ld_f(qt + i));
    if (h % G == 0)
        for (int i = tid; i < D; i += 256) {
            Kc[(int64_t)pos * D + i] = kt[i];
            Vc[(int64_t)pos * D + i] = vt[i];
        }

    // ---- local causal attention over keys 0..pos ----
    float qr[PL], o[PL];
#pragma unroll
    for (int e = 0; e < PL; ++e) {
        qr[e] = ld_f(qt + lane + 32 * e);
        o[e] = 0.f;
    }
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;   // softmax scale * log2(e)
    float m = -INFINITY, l = 0.f;
    for (int j = warp; j <= pos; j += NW) {
        const T *kr = j == pos ? kt : Kc + (int64_t)j * D;
        const T *vr = j == pos ? vt : Vc + (int64_t)j * D;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < PL; ++e) part = fmaf(qr[e], ld_f(kr + lane + 32 * e), part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        const float x = part * sl2;
        const float mn = fmaxf(m, x);
        const float a = exp2f(m - mn), p = exp2f(x - mn);   // a = 0 on the first key
        l = l * a + p;
#pragma unroll
        for (int e = 0; e < PL; ++e) o[e] = fmaf(p, ld_f(vr + lane + 32 * e), o[e] * a);
        m = mn;
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
#pragma unroll
    for (int e = 0; e < PL; ++e) s_o[warp][lane + 32 * e] = o[e];
    __syncthreads();

    // ---- retrieval: partial sums of sigma(q) M over PARTS row blocks; den by warp 0 ----
    {
        const int c = tid % D, part = tid / D;
        const float *Mc = M + chain * D * D + (int64_t)(part * FP) * D + c;
        float acc = 0.f;
#pragma unroll 8
        for (int f = 0; f < FP; ++f) acc = fmaf(s_sq[part * FP + f], Mc[(int64_t)f * D], acc);
        s_num[part][c] = acc;
    }
    if (warp == 0) {
        float part = 0.f;
        for (int f = lane; f < D; f += 32) part = fmaf(s_sq[f], z[chain * D + f], part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) s_den = part;
    }
    __syncthreads();

    if (tid < D) {
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) mx = fmaxf(mx, s_m[w]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float sc = exp2f(s_m[w] - mx);   // 0 for a warp that saw no key
            lsum = fmaf(s_l[w], sc, lsum);
            osum = fmaf(s_o[w][tid], sc, osum);
        }
        float num = 0.f;
#pragma unroll
        for (int pp = 0; pp < PARTS; ++pp) num += s_num[pp][tid];
        const float den = s_den;
        const float amem = den == 0.f ? 0.f : num / den;
        const float g = 1.f / (1.f + expf(-beta[h]));
        st_f(out + bh * D + tid, g * amem + (1.f - g) * (osum / lsum));
    }
}

}  // namespace infini
