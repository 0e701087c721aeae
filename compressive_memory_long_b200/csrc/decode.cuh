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

#include "simt_kernels.cuh"

namespace infini {

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
