// Backward pass of the Infini-attention forward (CUDA cores, fp32 arithmetic).
//
// Gradients of  <dout, out> + <dM, M_out> + <dz, z_out>  with respect to q, k, v, beta, M0
// and z0, through every path of the forward (AI Wiki "Infini-Attention", "What happens
// inside the Infini-attention block?", "How does the compressive memory work?"; the
// gradients flow through the memory recurrence as in "How is an Infini-attention model
// trained?").  Per segment s of a chain, with g = sigmoid(beta_h), dA_dot = (1 - g) dout
// and dA_mem = g dout:
//   local attention (causal softmax within the segment): the usual recomputation form,
//     P = exp(S - lse), D_i = dA_dot_i . A_dot_i, dS = P * (dA_dot V^T - D),
//     dq += dS K / sqrt(d), dk += dS^T Q / sqrt(d), dv += P^T dA_dot;
//   retrieval A_mem = num / den, num = sigma(q) M_{s-1}, den = sigma(q) . z_{s-1} (0 and no
//     gradient where den = 0): dnum = dA_mem / den, dden = -(dA_mem . A_mem) / den,
//     dsigma(q) = dnum M^T + dden z, and the memory before the segment receives
//     G^M_s = sum sigma(q)^T dnum, G^z_s = sum sigma(q) dden (over the group's heads);
//   gate: dbeta_h += g (1 - g) dout . (A_mem - A_dot);
//   memory update, with dM_s / dz_s the gradient of the memory after segment s:
//     linear: dM_{s-1} = dM_s + G^M_s, dsigma(k_t) += dM_s v_t, dv_t += sigma(k_t) dM_s;
//     delta:  dM_{s-1} = dM_s - A_s dM_s + G^M_s with A_s = sigma(K)^T diag(1/den) sigma(K),
//             den_t = sigma(k_t) . z_{s-1}; with R_t = sigma(k_t) M_{s-1} / den_t,
//             U_t = v_t - R_t, dU_t = sigma(k_t) dM_s: dv_t += dU_t,
//             dsigma(k_t) += dM_s U_t - M_{s-1} dU_t / den_t + dden_t z_{s-1},
//             dden_t = (dU_t . R_t) / den_t, and dz_{s-1} receives sum_t dden_t sigma(k_t);
//     both:   dz_{s-1} += dz_s, dsigma(k_t) += dz_s;
//   dk = dsigma(k) * sigma'(k), dq += dsigma(q) * sigma'(q), sigma'(x) = 1 (x > 0), e^x.
// dM0 = dM_{-1}, dz0 = dz_{-1}.
//
// Kernels, in launch order (workspace fp32; slots as the forward's snapshots, a short last
// segment being one more slot):
//   k_bwd_rows    per (b, h, segment, 64 query rows): recomputes the forward of the rows and
//                 writes lse, D, the retrieval's row factors, the retrieval part of dq and
//                 the gate's partial sums
//   k_bwd_dq      per (b, h, segment, 64 query rows): dq = retrieval part + local part
//   k_bwd_dkdv    per (b, kv head, segment, 64 keys): local dk, dv over the group's heads
//   k_bwd_gm      per (chain, segment): G^M_s, G^z_s
//   k_bwd_mlin / k_bwd_mdelta  the reverse memory recurrence: dM_s of every segment, dM0
//   k_bwd_update  per (chain, segment): the update's dsigma(k), dv and h_s
//   k_bwd_zrev    the reverse z recurrence: dz_s of every segment, dz0
//   k_bwd_final   dk, dv in the activation dtype; k_bwd_beta the gate's gradient
#pragma once

#include "simt_kernels.cuh"

namespace infini {

__device__ __forceinline__ float sigma_grad(float x) { return x > 0.f ? 1.f : expf(x); }

struct BwdWs {
    const float *snapM, *snapZ;   // [chains * S, D, D], [chains * S, D]: M_{s-1}, z_{s-1}
    float *lse;                   // [B, H, L]: row max * log2(e) / sqrt(d) + log2(row sum)
    float *Drow;                  // [B, H, L]: dA_dot . A_dot
    float *wsc;                   // [B, H, L]: g / den (0 where den = 0)
    float *dden;                  // [B, H, L]: the retrieval's dden
    float *dq;                    // [B, H, L, D]: the retrieval part of dq
    float *dbeta_part;            // [B, H, S, qtiles]
    float *dk, *dv;               // [B, Hkv, L, D]: local parts, then dv += the update's
    float *dsk;                   // [B, Hkv, L, D]: the update's dsigma(k) (without dz_s)
    float *GM, *Gz;               // [chains * S, D, D], [chains * S, D]
    float *dMs;                   // [chains * S, D, D]: dM_s, gradient of M after segment s
    float *h;                     // [chains * S, D]
    float *dzs;                   // [chains * S, D]: dz_s
};

// ---------------------------------------------------------------------------------------
// Row statistics: the forward of 64 query rows (local attention with an online softmax,
// retrieval, gate), then per row lse, D = dA_dot . A_dot, the retrieval factors
// wsc = g / den and dden = -g (dout . A_mem) / den, the retrieval part of dq and the
// gate's partial sum.  Same tiling as k_segment_simt.
// ---------------------------------------------------------------------------------------
template <int D>
struct BwdRowsSmem {
    static constexpr int BQ = 64, BK = 64;
    static constexpr int floats = 2 * BQ * (D + 1) + BK * (D + 1) + BK * D + BQ * (BK + 1);
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_rows(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
           const float *__restrict__ beta, const T *__restrict__ dout, BwdWs w, int64_t L,
           int N, int S, int H, int Hkv)
{
    constexpr int BQ = 64, BK = 64, RJ = D / 16;
    extern __shared__ float smem[];
    float *sQ = smem;                    // [BQ][D+1]
    float *sO = sQ + BQ * (D + 1);       // [BQ][D+1]: dout rows
    float *sK = sO + BQ * (D + 1);       // [BK][D+1]
    float *sV = sK + BK * (D + 1);       // [BK][D]
    float *sP = sV + BK * D;             // [BQ][BK+1]

    const int qtiles = (N + BQ - 1) / BQ;
    int64_t bid = blockIdx.x;
    const int qt = (int)(bid % qtiles); bid /= qtiles;
    const int s = (int)(bid % S); bid /= S;
    const int64_t bh = bid;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int64_t chain = b * Hkv + h / (H / Hkv);
    const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
    const int q0 = qt * BQ;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    float *part = w.dbeta_part + (bh * S + s) * qtiles + qt;
    if (q0 >= valid) {
        if (tid == 0) *part = 0.f;
        return;
    }
    const int64_t tok0 = (int64_t)s * N + q0;
    const T *Q = q + (bh * L + tok0) * D;
    const T *dO = dout + (bh * L + tok0) * D;
    const T *Kseg = k + (chain * L + (int64_t)s * N) * D;
    const T *Vseg = v + (chain * L + (int64_t)s * N) * D;
    for (int i = tid; i < BQ * D; i += 256) {
        const bool in = q0 + i / D < valid;
        sQ[(i / D) * (D + 1) + i % D] = in ? ld_f(Q + i) : 0.f;
        sO[(i / D) * (D + 1) + i % D] = in ? ld_f(dO + i) : 0.f;
    }

    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    float m[4], l[4], o[4][RJ];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int j = 0; j < RJ; ++j) o[i][j] = 0.f;
    }
    for (int kt = 0; kt <= qt; ++kt) {
        __syncthreads();
        const T *Kt = Kseg + (int64_t)kt * BK * D;
        const T *Vt = Vseg + (int64_t)kt * BK * D;
        for (int i = tid; i < BK * D; i += 256) {
            const bool in = kt * BK + i / D < valid;
            sK[(i / D) * (D + 1) + i % D] = in ? ld_f(Kt + i) : 0.f;
            sV[i] = in ? ld_f(Vt + i) : 0.f;
        }
        __syncthreads();
        float sc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll 4
        for (int c = 0; c < D; ++c) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = sQ[(ty + 16 * i) * (D + 1) + c];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = sK[(tx + 16 * j) * (D + 1) + c];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sc[i][j] = fmaf(a[i], bb[j], sc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 16 * i;
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = tx + 16 * j;
                float x = sc[i][j] * sl2;
                if ((kt == qt && c > r) || kt * BK + c >= valid) x = -INFINITY;
                sc[i][j] = x;
                mx = fmaxf(mx, x);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mnew = fmaxf(m[i], mx);
            const float alpha = exp2f(m[i] - mnew);
            float rs = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float p = exp2f(sc[i][j] - mnew);
                rs += p;
                sP[r * (BK + 1) + tx + 16 * j] = p;
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
            l[i] = l[i] * alpha + rs;
            m[i] = mnew;
#pragma unroll
            for (int j = 0; j < RJ; ++j) o[i][j] *= alpha;
        }
        __syncthreads();
#pragma unroll 4
        for (int kv = 0; kv < BK; ++kv) {
            float vv[RJ];
#pragma unroll
            for (int j = 0; j < RJ; ++j) vv[j] = sV[kv * D + tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float p = sP[(ty + 16 * i) * (BK + 1) + kv];
#pragma unroll
                for (int j = 0; j < RJ; ++j) o[i][j] = fmaf(p, vv[j], o[i][j]);
            }
        }
    }
    // ---- retrieval: num = sigma(q) M, den = sigma(q) . z; and dO M^T for dsigma(q)
    __syncthreads();
    float *sS = sK;                      // sigma(q) rows [BQ][D+1] (the K tile's room)
    for (int i = tid; i < BQ * D; i += 256) {
        const int r = i / D, c = i % D;
        sS[r * (D + 1) + c] = feature_map(sQ[r * (D + 1) + c]);
    }
    const float *Ms = w.snapM + (chain * S + s) * (int64_t)D * D;
    const float *zs = w.snapZ + (chain * S + s) * (int64_t)D;
    float *sZ = sP;                      // z_{s-1}
    for (int i = tid; i < D; i += 256) sZ[i] = zs[i];
    __syncthreads();
    float den[4], num[4][RJ], dom[4][RJ];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a = 0.f;
        for (int c = 0; c < D; ++c) a = fmaf(sS[(ty + 16 * i) * (D + 1) + c], sZ[c], a);
        den[i] = a;
#pragma unroll
        for (int j = 0; j < RJ; ++j) num[i][j] = dom[i][j] = 0.f;
    }
    float *sMc = sV;                     // 32 rows of M at a time [32][D+1] (fits BK * D)
    for (int kc = 0; kc < D; kc += 32) {
        __syncthreads();
        for (int i = tid; i < 32 * D; i += 256) sMc[(i / D) * (D + 1) + i % D] = Ms[(int64_t)kc * D + i];
        __syncthreads();
        // num[r][c] += sum_kk sigma(q)[r][kc+kk] M[kc+kk][c]
#pragma unroll 4
        for (int kk = 0; kk < 32; ++kk) {
            float mm[RJ];
#pragma unroll
            for (int j = 0; j < RJ; ++j) mm[j] = sMc[kk * (D + 1) + tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = sS[(ty + 16 * i) * (D + 1) + kc + kk];
#pragma unroll
                for (int j = 0; j < RJ; ++j) num[i][j] = fmaf(a, mm[j], num[i][j]);
            }
        }
        // dom[r][a] (a = kc + kk in this chunk, for this thread's a's) = sum_c dO[r][c] M[a][c]
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
            const int aa = tx + 16 * j;
            if (aa < kc || aa >= kc + 32) continue;
            for (int c = 0; c < D; ++c) {
                const float mv = sMc[(aa - kc) * (D + 1) + c];
#pragma unroll
                for (int i = 0; i < 4; ++i) dom[i][j] = fmaf(sO[(ty + 16 * i) * (D + 1) + c], mv, dom[i][j]);
            }
        }
    }
    const float g = 1.f / (1.f + expf(-beta[h]));
    float gpart = 0.f;
    const int64_t row0 = bh * L + tok0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        const float inv_l = 1.f / l[i];
        float dd = 0.f, gm = 0.f, dam = 0.f;      // dO . A_dot, dO . (A_mem - A_dot), dO . A_mem
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
            const float adot = o[i][j] * inv_l;
            const float amem = den[i] == 0.f ? 0.f : num[i][j] / den[i];
            const float d0 = sO[r * (D + 1) + tx + 16 * j];
            dd = fmaf(d0, adot, dd);
            dam = fmaf(d0, amem, dam);
            gm = fmaf(d0, amem - adot, gm);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {
            dd += __shfl_xor_sync(0xffffffffu, dd, off);
            dam += __shfl_xor_sync(0xffffffffu, dam, off);
            gm += __shfl_xor_sync(0xffffffffu, gm, off);
        }
        const bool live = q0 + r < valid;
        const float ws = den[i] == 0.f ? 0.f : g / den[i];
        const float ddn = den[i] == 0.f ? 0.f : -g * dam / den[i];
        if (live) {
            gpart += tx == 0 ? gm : 0.f;
            if (tx == 0) {
                w.lse[row0 + r] = m[i] + log2f(l[i]);
                w.Drow[row0 + r] = (1.f - g) * dd;
                w.wsc[row0 + r] = ws;
                w.dden[row0 + r] = ddn;
            }
            // dq (retrieval part) = (wsc dO M^T + dden z) * sigma'(q)
#pragma unroll
            for (int j = 0; j < RJ; ++j) {
                const int a = tx + 16 * j;
                const float ds = fmaf(ws, dom[i][j], ddn * sZ[a]);
                w.dq[(row0 + r) * D + a] = ds * sigma_grad(sQ[r * (D + 1) + a]);
            }
        }
    }
    // the gate's partial sum over this tile's rows, in a fixed order
    __syncthreads();
    float *red = sP;
    if (tx == 0) red[ty] = gpart;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int i = 0; i < 16; ++i) t += red[i];
        *part = g * (1.f - g) * t;
    }
}

// ---------------------------------------------------------------------------------------
// dq = retrieval part + sum_j dS_ij k_j / sqrt(d) over keys j <= i of the segment, with
// P recomputed from lse and dS = P (dA_dot . v_j - D_i).
// ---------------------------------------------------------------------------------------
template <int D>
struct BwdDqSmem {
    static constexpr int BQ = 64, BK = 64;
    static constexpr int floats = 2 * BQ * (D + 1) + 2 * BK * (D + 1) + BQ * (BK + 1);
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_dq(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
         const float *__restrict__ beta, const T *__restrict__ dout, BwdWs w, T *__restrict__ dq,
         int64_t L, int N, int S, int H, int Hkv)
{
    constexpr int BQ = 64, BK = 64, RJ = D / 16;
    extern __shared__ float smem[];
    float *sQ = smem;                    // [BQ][D+1]
    float *sA = sQ + BQ * (D + 1);       // [BQ][D+1]: dA_dot = (1 - g) dout
    float *sK = sA + BQ * (D + 1);       // [BK][D+1]
    float *sV = sK + BK * (D + 1);       // [BK][D+1]
    float *sP = sV + BK * (D + 1);       // [BQ][BK+1]: dS

    const int qtiles = (N + BQ - 1) / BQ;
    int64_t bid = blockIdx.x;
    const int qt = (int)(bid % qtiles); bid /= qtiles;
    const int s = (int)(bid % S); bid /= S;
    const int64_t bh = bid;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int64_t chain = b * Hkv + h / (H / Hkv);
    const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
    const int q0 = qt * BQ;
    if (q0 >= valid) return;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int64_t tok0 = (int64_t)s * N + q0, row0 = bh * L + tok0;
    const float g = 1.f / (1.f + expf(-beta[h]));
    for (int i = tid; i < BQ * D; i += 256) {
        const bool in = q0 + i / D < valid;
        sQ[(i / D) * (D + 1) + i % D] = in ? ld_f(q + row0 * D + i) : 0.f;
        sA[(i / D) * (D + 1) + i % D] = in ? (1.f - g) * ld_f(dout + row0 * D + i) : 0.f;
    }
    float lse[4], Dr[4], acc[4][RJ];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        const bool in = q0 + r < valid;
        lse[i] = in ? w.lse[row0 + r] : 0.f;
        Dr[i] = in ? w.Drow[row0 + r] : 0.f;
#pragma unroll
        for (int j = 0; j < RJ; ++j) acc[i][j] = 0.f;
    }
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    const T *Kseg = k + (chain * L + (int64_t)s * N) * D;
    const T *Vseg = v + (chain * L + (int64_t)s * N) * D;
    for (int kt = 0; kt <= qt; ++kt) {
        __syncthreads();
        for (int i = tid; i < BK * D; i += 256) {
            const bool in = kt * BK + i / D < valid;
            sK[(i / D) * (D + 1) + i % D] = in ? ld_f(Kseg + (int64_t)kt * BK * D + i) : 0.f;
            sV[(i / D) * (D + 1) + i % D] = in ? ld_f(Vseg + (int64_t)kt * BK * D + i) : 0.f;
        }
        __syncthreads();
        float sc[4][4], dp[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) sc[i][j] = dp[i][j] = 0.f;
#pragma unroll 4
        for (int c = 0; c < D; ++c) {
            float a[4], da[4], bk[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = sQ[(ty + 16 * i) * (D + 1) + c];
                da[i] = sA[(ty + 16 * i) * (D + 1) + c];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bk[j] = sK[(tx + 16 * j) * (D + 1) + c];
                bv[j] = sV[(tx + 16 * j) * (D + 1) + c];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sc[i][j] = fmaf(a[i], bk[j], sc[i][j]);
                    dp[i][j] = fmaf(da[i], bv[j], dp[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 16 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = tx + 16 * j;
                const bool vis = !(kt == qt && c > r) && kt * BK + c < valid && q0 + r < valid;
                const float p = vis ? exp2f(sc[i][j] * sl2 - lse[i]) : 0.f;
                sP[r * (BK + 1) + c] = p * (dp[i][j] - Dr[i]);
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int kv = 0; kv < BK; ++kv) {
            float kk[RJ];
#pragma unroll
            for (int j = 0; j < RJ; ++j) kk[j] = sK[kv * (D + 1) + tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float d = sP[(ty + 16 * i) * (BK + 1) + kv];
#pragma unroll
                for (int j = 0; j < RJ; ++j) acc[i][j] = fmaf(d, kk[j], acc[i][j]);
            }
        }
    }
    const float rs = rsqrtf((float)D);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        if (q0 + r >= valid) continue;
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
            const int a = tx + 16 * j;
            st_f(dq + (row0 + r) * D + a, w.dq[(row0 + r) * D + a] + acc[i][j] * rs);
        }
    }
}

// ---------------------------------------------------------------------------------------
// dk, dv of 64 keys of a segment from the local attention of every query head of the group
// and every query row at or after them: dv_j = sum_i P_ij dA_dot_i,
// dk_j = sum_i dS_ij q_i / sqrt(d).  Each key row has one owner: no atomics.
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_dkdv(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
           const float *__restrict__ beta, const T *__restrict__ dout, BwdWs w, int64_t L, int N,
           int S, int H, int Hkv)
{
    constexpr int BQ = 64, BK = 64, RJ = D / 16;
    extern __shared__ float smem[];
    float *sK = smem;                    // [BK][D+1]
    float *sV = sK + BK * (D + 1);       // [BK][D+1]
    float *sQ = sV + BK * (D + 1);       // [BQ][D+1]
    float *sA = sQ + BQ * (D + 1);       // [BQ][D+1]
    float *sP = sA + BQ * (D + 1);       // [BK][BQ+1]: P^T, then dS^T

    const int ktiles = (N + BK - 1) / BK;
    int64_t bid = blockIdx.x;
    const int kt = (int)(bid % ktiles); bid /= ktiles;
    const int s = (int)(bid % S); bid /= S;
    const int64_t chain = bid;           // b * Hkv + kvh
    const int kvh = (int)(chain % Hkv);
    const int64_t b = chain / Hkv;
    const int G = H / Hkv;
    const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
    const int k0 = kt * BK;
    if (k0 >= valid) return;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int64_t krow0 = chain * L + (int64_t)s * N + k0;
    for (int i = tid; i < BK * D; i += 256) {
        const bool in = k0 + i / D < valid;
        sK[(i / D) * (D + 1) + i % D] = in ? ld_f(k + krow0 * D + i) : 0.f;
        sV[(i / D) * (D + 1) + i % D] = in ? ld_f(v + krow0 * D + i) : 0.f;
    }
    // thread (ty, tx) owns keys ty + 16 i and output columns tx + 16 j
    float dk[4][RJ], dv[4][RJ];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < RJ; ++j) dk[i][j] = dv[i][j] = 0.f;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    for (int gq = 0; gq < G; ++gq) {
        const int h = kvh * G + gq;
        const int64_t bh = b * H + h;
        const float g = 1.f / (1.f + expf(-beta[h]));
        for (int qt = kt; qt * BQ < valid; ++qt) {
            const int q0 = qt * BQ;
            const int64_t row0 = bh * L + (int64_t)s * N + q0;
            __syncthreads();
            for (int i = tid; i < BQ * D; i += 256) {
                const bool in = q0 + i / D < valid;
                sQ[(i / D) * (D + 1) + i % D] = in ? ld_f(q + row0 * D + i) : 0.f;
                sA[(i / D) * (D + 1) + i % D] = in ? (1.f - g) * ld_f(dout + row0 * D + i) : 0.f;
            }
            __syncthreads();
            // scores and dP for keys ty + 16 i (rows of the transposed tile), queries tx + 16 j
            float sc[4][4], dp[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sc[i][j] = dp[i][j] = 0.f;
#pragma unroll 4
            for (int c = 0; c < D; ++c) {
                float kk[4], vv[4], qq[4], aa[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    kk[i] = sK[(ty + 16 * i) * (D + 1) + c];
                    vv[i] = sV[(ty + 16 * i) * (D + 1) + c];
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qq[j] = sQ[(tx + 16 * j) * (D + 1) + c];
                    aa[j] = sA[(tx + 16 * j) * (D + 1) + c];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        sc[i][j] = fmaf(kk[i], qq[j], sc[i][j]);
                        dp[i][j] = fmaf(vv[i], aa[j], dp[i][j]);
                    }
            }
            float pt[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int qi = tx + 16 * j;
                const bool qin = q0 + qi < valid;
                const float lse = qin ? w.lse[row0 + qi] : 0.f;
                const float Dr = qin ? w.Drow[row0 + qi] : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kj = ty + 16 * i;
                    const bool vis = qin && k0 + kj < valid && q0 + qi >= k0 + kj;
                    const float p = vis ? exp2f(sc[i][j] * sl2 - lse) : 0.f;
                    pt[i][j] = p;
                    dp[i][j] = p * (dp[i][j] - Dr);          // dS^T
                }
            }
            // dv += P^T dA (contraction over the 64 queries)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sP[(ty + 16 * i) * (BQ + 1) + tx + 16 * j] = pt[i][j];
            __syncthreads();
#pragma unroll 4
            for (int qi = 0; qi < BQ; ++qi) {
                float av[RJ];
#pragma unroll
                for (int j = 0; j < RJ; ++j) av[j] = sA[qi * (D + 1) + tx + 16 * j];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float p = sP[(ty + 16 * i) * (BQ + 1) + qi];
#pragma unroll
                    for (int j = 0; j < RJ; ++j) dv[i][j] = fmaf(p, av[j], dv[i][j]);
                }
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sP[(ty + 16 * i) * (BQ + 1) + tx + 16 * j] = dp[i][j];
            __syncthreads();
#pragma unroll 4
            for (int qi = 0; qi < BQ; ++qi) {
                float qv[RJ];
#pragma unroll
                for (int j = 0; j < RJ; ++j) qv[j] = sQ[qi * (D + 1) + tx + 16 * j];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float d = sP[(ty + 16 * i) * (BQ + 1) + qi];
#pragma unroll
                    for (int j = 0; j < RJ; ++j) dk[i][j] = fmaf(d, qv[j], dk[i][j]);
                }
            }
        }
    }
    const float rs = rsqrtf((float)D);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kj = ty + 16 * i;
        if (k0 + kj >= valid) continue;
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
            const int a = tx + 16 * j;
            w.dk[(krow0 + kj) * D + a] = dk[i][j] * rs;
            w.dv[(krow0 + kj) * D + a] = dv[i][j];
        }
    }
}

// ---------------------------------------------------------------------------------------
// G^M_s = sum over the group's heads and the segment's rows of sigma(q)^T (wsc dout) and
// G^z_s = sum sigma(q) dden.  One CTA per (chain, segment); thread (ty, tx) owns rows
// ty + 16 i and columns tx + 16 j of G^M.
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_gm(const T *__restrict__ q, const T *__restrict__ dout, BwdWs w, int64_t L, int N, int S,
         int H, int Hkv)
{
    constexpr int TK = 32, R = D / 16;
    __shared__ float sS[TK][D + 1];      // sigma(q) rows
    __shared__ float sW[TK][D + 1];      // wsc dout rows
    __shared__ float sDd[TK];
    const int64_t cs = blockIdx.x;
    const int64_t chain = cs / S;
    const int s = (int)(cs % S);
    const int kvh = (int)(chain % Hkv);
    const int64_t b = chain / Hkv;
    const int G = H / Hkv;
    const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    float acc[R][R];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = 0.f;
    float zacc = 0.f;
    for (int gq = 0; gq < G; ++gq) {
        const int64_t row0 = (b * H + kvh * G + gq) * L + (int64_t)s * N;
        for (int t0 = 0; t0 < valid; t0 += TK) {
            __syncthreads();
            for (int i = tid; i < TK * D; i += 256) {
                const int t = i / D, c = i % D;
                const bool in = t0 + t < valid;
                sS[t][c] = in ? feature_map(ld_f(q + (row0 + t0 + t) * D + c)) : 0.f;
                sW[t][c] = in ? w.wsc[row0 + t0 + t] * ld_f(dout + (row0 + t0 + t) * D + c) : 0.f;
            }
            if (tid < TK) sDd[tid] = t0 + tid < valid ? w.dden[row0 + t0 + tid] : 0.f;
            __syncthreads();
#pragma unroll 4
            for (int t = 0; t < TK; ++t) {
                float a[R], bb[R];
#pragma unroll
                for (int i = 0; i < R; ++i) a[i] = sS[t][ty + 16 * i];
#pragma unroll
                for (int j = 0; j < R; ++j) bb[j] = sW[t][tx + 16 * j];
#pragma unroll
                for (int i = 0; i < R; ++i)
#pragma unroll
                    for (int j = 0; j < R; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
            }
            if (tid < D)
                for (int t = 0; t < TK; ++t) zacc = fmaf(sS[t][tid], sDd[t], zacc);
        }
    }
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) w.GM[(cs * D + ty + 16 * i) * D + tx + 16 * j] = acc[i][j];
    if (tid < D) w.Gz[cs * D + tid] = zacc;
}

// ---------------------------------------------------------------------------------------
// Reverse memory recurrence, additive rule: dM_{s-1} = dM_s + G^M_s from dM_{S-1} = dM.
// One thread per element; dMs[s] = dM_s; dM0 = dM_{-1}.  The loads of G^M run eight
// segments ahead of the dependent sums (G^M and dMs never overlap), so a thread keeps eight
// memory reads in flight instead of one.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_bwd_mlin(const float *dM, BwdWs w, float *dM0, int S, int D, int64_t chains)
{
    const int64_t DD = (int64_t)D * D;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= chains * DD) return;
    const int64_t chain = i / DD, e = i % DD;
    const float *__restrict__ gm = w.GM + chain * S * DD + e;
    float *__restrict__ out = w.dMs + chain * S * DD + e;
    float m = dM ? dM[i] : 0.f;
    int s = S - 1;
    for (; s >= 7; s -= 8) {
        float g[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) g[u] = gm[(int64_t)(s - u) * DD];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            out[(int64_t)(s - u) * DD] = m;
            m += g[u];
        }
    }
    for (; s >= 0; --s) {
        out[(int64_t)s * DD] = m;
        m += gm[(int64_t)s * DD];
    }
    if (dM0) dM0[i] = m;
}

// ---------------------------------------------------------------------------------------
// Reverse memory recurrence, delta rule: dM_{s-1} = dM_s - sigma(K)^T diag(1/den)
// (sigma(K) dM_s) + G^M_s, segments in reverse order.  Column block e of dM_{s-1} needs
// only column block e of dM_s (the same structure as the forward chain), so each CTA owns
// CB columns of one chain and keeps them in shared memory.  dMs[s] = dM_s; dM0 = dM_{-1}.
// ---------------------------------------------------------------------------------------
template <typename T, int D, int CB>
__global__ void __launch_bounds__(256)
k_bwd_mdelta(const T *__restrict__ k, const float *dM, BwdWs w, float *dM0, int64_t L, int N,
             int S)
{
    constexpr int TK = 32, NBLK = D / CB, PER = D * CB / 256;
    static_assert(PER >= 1 && (D * CB) % 256 == 0, "column block too small");
    __shared__ float sM[D][CB];
    __shared__ float sz[D];
    __shared__ float sK[TK][D + 1];
    __shared__ float sU[TK][CB];
    __shared__ float sden[TK];
    const int64_t chain = blockIdx.x / NBLK;
    const int cb = (blockIdx.x % NBLK) * CB;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    for (int i = tid; i < D * CB; i += 256)
        sM[i / CB][i % CB] = dM ? dM[(chain * D + i / CB) * D + cb + i % CB] : 0.f;
    __syncthreads();
    for (int s = S - 1; s >= 0; --s) {
        const int64_t slot = chain * S + s;
        for (int i = tid; i < D * CB; i += 256)
            w.dMs[(slot * D + i / CB) * D + cb + i % CB] = sM[i / CB][i % CB];
        for (int i = tid; i < D; i += 256) sz[i] = w.snapZ[slot * D + i];
        const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
        const T *K = k + (chain * L + (int64_t)s * N) * D;
        float dm[PER];
#pragma unroll
        for (int p = 0; p < PER; ++p) dm[p] = 0.f;
        __syncthreads();
        for (int t0 = 0; t0 < valid; t0 += TK) {
            for (int i = tid; i < TK * D; i += 256) {
                const int t = i / D, c = i % D;
                sK[t][c] = t0 + t < valid ? feature_map(ld_f(K + (int64_t)(t0 + t) * D + c)) : 0.f;
            }
            __syncthreads();
            for (int t = warp; t < TK; t += 8) {
                float part = 0.f;
                for (int c = lane; c < D; c += 32) part = fmaf(sK[t][c], sz[c], part);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) sden[t] = part;
            }
            __syncthreads();
            // U = -sigma(K) dM_s / den  (0 where den == 0)
            for (int i = tid; i < TK * CB; i += 256) {
                const int t = i / CB, e = i % CB;
                float r = 0.f;
#pragma unroll 8
                for (int c = 0; c < D; ++c) r = fmaf(sK[t][c], sM[c][e], r);
                const float den = sden[t];
                sU[t][e] = den == 0.f ? 0.f : -r / den;
            }
            __syncthreads();
#pragma unroll
            for (int p = 0; p < PER; ++p) {
                const int i = tid + 256 * p, c = i / CB, e = i % CB;
                float a = dm[p];
#pragma unroll 8
                for (int t = 0; t < TK; ++t) a = fmaf(sK[t][c], sU[t][e], a);
                dm[p] = a;
            }
            __syncthreads();
        }
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            const int i = tid + 256 * p, c = i / CB, e = i % CB;
            sM[c][e] += dm[p] + w.GM[(slot * D + c) * D + cb + e];
        }
        __syncthreads();
    }
    if (dM0)
        for (int i = tid; i < D * CB; i += 256)
            dM0[(chain * D + i / CB) * D + cb + i % CB] = sM[i / CB][i % CB];
}

// ---------------------------------------------------------------------------------------
// The update's gradients of one (chain, segment), token by token, from dM_s, M_{s-1} and
// z_{s-1}: dv += sigma(k) dM_s (linear) or dU (delta), dsk = dsigma(k) without the dz_s
// term, and h_s = sum_t dden_t sigma(k_t) (delta).  dM_s and M_{s-1} in shared memory.
// ---------------------------------------------------------------------------------------
template <int D>
struct BwdUpdSmem {
    static constexpr int TK = 32;
    static constexpr int floats = 2 * D * (D + 1) + 4 * TK * (D + 1) + D + 2 * TK;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename T, int D, bool DELTA>
__global__ void __launch_bounds__(256)
k_bwd_update(const T *__restrict__ k, const T *__restrict__ v, BwdWs w, int64_t L, int N, int S)
{
    constexpr int TK = 32, R = D / 16;
    extern __shared__ float smem[];
    float *sG = smem;                    // dM_s [D][D+1]
    float *sM = sG + D * (D + 1);        // M_{s-1} [D][D+1]
    float *sK = sM + D * (D + 1);        // sigma(k) [TK][D+1]
    float *sV = sK + TK * (D + 1);       // v [TK][D+1]
    float *sR = sV + TK * (D + 1);       // R_t [TK][D+1]
    float *sU = sR + TK * (D + 1);       // dU_t [TK][D+1]
    float *sz = sU + TK * (D + 1);       // z_{s-1}
    float *sden = sz + D;                // den_t
    float *sdd = sden + TK;              // dden_t
    const int64_t cs = blockIdx.x;
    const int64_t chain = cs / S;
    const int s = (int)(cs % S);
    const int valid = (int)(L - (int64_t)s * N < N ? L - (int64_t)s * N : N);
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16, warp = tid / 32, lane = tid % 32;
    for (int i = tid; i < D * D; i += 256) {
        sG[(i / D) * (D + 1) + i % D] = w.dMs[cs * D * D + i];
        if (DELTA) sM[(i / D) * (D + 1) + i % D] = w.snapM[cs * D * D + i];
    }
    for (int i = tid; i < D; i += 256) sz[i] = w.snapZ[cs * D + i];
    float hacc = 0.f;
    const int64_t rowbase = chain * L + (int64_t)s * N;
    for (int t0 = 0; t0 < valid; t0 += TK) {
        __syncthreads();
        for (int i = tid; i < TK * D; i += 256) {
            const int t = i / D, c = i % D;
            const bool in = t0 + t < valid;
            sK[t * (D + 1) + c] = in ? feature_map(ld_f(k + (rowbase + t0 + t) * D + c)) : 0.f;
            sV[t * (D + 1) + c] = in ? ld_f(v + (rowbase + t0 + t) * D + c) : 0.f;
        }
        __syncthreads();
        if (DELTA)
            for (int t = warp; t < TK; t += 8) {
                float part = 0.f;
                for (int c = lane; c < D; c += 32) part = fmaf(sK[t * (D + 1) + c], sz[c], part);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) sden[t] = part;
            }
        __syncthreads();
        // row products over the features: dU_t = sigma(k_t) dM_s and R_t = sigma(k_t) M / den
        // for tokens t = ty, ty + 16 and columns tx + 16 j
        for (int tt = ty; tt < TK; tt += 16) {
            float du[R], rr[R];
#pragma unroll
            for (int j = 0; j < R; ++j) du[j] = rr[j] = 0.f;
            for (int c = 0; c < D; ++c) {
                const float kc = sK[tt * (D + 1) + c];
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    du[j] = fmaf(kc, sG[c * (D + 1) + tx + 16 * j], du[j]);
                    if (DELTA) rr[j] = fmaf(kc, sM[c * (D + 1) + tx + 16 * j], rr[j]);
                }
            }
            const float den = DELTA ? sden[tt] : 0.f;
#pragma unroll
            for (int j = 0; j < R; ++j) {
                sU[tt * (D + 1) + tx + 16 * j] = du[j];
                if (DELTA) sR[tt * (D + 1) + tx + 16 * j] = den == 0.f ? 0.f : rr[j] / den;
            }
        }
        __syncthreads();
        // dden_t = (dU_t . R_t) / den_t
        if (DELTA)
            for (int t = warp; t < TK; t += 8) {
                float part = 0.f;
                for (int c = lane; c < D; c += 32) part = fmaf(sU[t * (D + 1) + c], sR[t * (D + 1) + c], part);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) sdd[t] = sden[t] == 0.f ? 0.f : part / sden[t];
            }
        __syncthreads();
        // column products: dsigma(k_t)[i] = sum_j dM[i][j] U_t[j] - sum_j M[i][j] dU_t[j] / den_t
        // + dden_t z[i]  (U_t = v_t - R_t; linear: sum_j dM[i][j] v_t[j]) for rows i = tx + 16 j
        for (int tt = ty; tt < TK; tt += 16) {
            const bool in = t0 + tt < valid;
            float ds[R];
#pragma unroll
            for (int j = 0; j < R; ++j) ds[j] = 0.f;
            const float den = DELTA ? sden[tt] : 0.f;
            const float inv = den == 0.f ? 0.f : 1.f / den;
            for (int c = 0; c < D; ++c) {
                const float u = DELTA ? sV[tt * (D + 1) + c] - sR[tt * (D + 1) + c] : sV[tt * (D + 1) + c];
                const float du = sU[tt * (D + 1) + c] * inv;
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    ds[j] = fmaf(sG[(tx + 16 * j) * (D + 1) + c], u, ds[j]);
                    if (DELTA) ds[j] = fmaf(-sM[(tx + 16 * j) * (D + 1) + c], du, ds[j]);
                }
            }
            if (in) {
                const int64_t row = rowbase + t0 + tt;
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    const int a = tx + 16 * j;
                    float val = ds[j];
                    if (DELTA) val = fmaf(sdd[tt], sz[a], val);
                    w.dsk[row * D + a] = val;
                    w.dv[row * D + a] += sU[tt * (D + 1) + a];     // dU_t (delta) = sigma(k_t) dM_s
                }
            }
        }
        if (DELTA && tid < D)
            for (int t = 0; t < TK; ++t) hacc = fmaf(sdd[t], sK[t * (D + 1) + tid], hacc);
    }
    if (tid < D) w.h[cs * D + tid] = DELTA ? hacc : 0.f;
}

// ---------------------------------------------------------------------------------------
// Reverse z recurrence: dz_{s-1} = dz_s + G^z_s + h_s from dz_{S-1} = dz; dzs[s] = dz_s;
// dz0 = dz_{-1}.  A block of 32 features x ZREV_CHUNKS threads per (chain, 32 features): each
// thread sums G^z + h over its chunk of consecutive segments, the chunk totals give every
// chunk its starting value (the sum over the later chunks), and each thread then walks its
// chunk backwards writing dz_s.  The summation order is fixed by the chunking.
// ---------------------------------------------------------------------------------------
constexpr int ZREV_CHUNKS = 32;

__global__ void __launch_bounds__(32 * ZREV_CHUNKS)
k_bwd_zrev(const float *dz, BwdWs w, float *dz0, int S, int D, int64_t chains)
{
    __shared__ float tot[ZREV_CHUNKS][32];
    const int fb = D / 32 > 0 ? D / 32 : 1;                 // 32-feature blocks per chain
    const int64_t chain = blockIdx.x / fb;
    const int f = (int)(blockIdx.x % fb) * 32 + (threadIdx.x & 31);
    const int c = threadIdx.x >> 5;
    const bool live = f < D;                                // d = 32: one block, all live
    const int len = (S + ZREV_CHUNKS - 1) / ZREV_CHUNKS;
    const int s0 = c * len, s1 = s0 + len < S ? s0 + len : S;
    const float *__restrict__ gz = w.Gz + chain * S * D + f;
    const float *__restrict__ hh = w.h + chain * S * D + f;
    float *__restrict__ out = w.dzs + chain * S * D + f;
    float t = 0.f;
    if (live)
        for (int s = s0; s < s1; ++s) t += gz[(int64_t)s * D] + hh[(int64_t)s * D];
    tot[c][threadIdx.x & 31] = t;
    __syncthreads();
    if (!live) return;
    float z = dz ? dz[chain * D + f] : 0.f;
    for (int j = ZREV_CHUNKS - 1; j > c; --j) z += tot[j][threadIdx.x & 31];
    for (int s = s1 - 1; s >= s0; --s) {
        out[(int64_t)s * D] = z;
        z += gz[(int64_t)s * D] + hh[(int64_t)s * D];
    }
    if (c == 0 && dz0) dz0[chain * D + f] = z;
}

// ---------------------------------------------------------------------------------------
// dk = (dsk + dz_s) sigma'(k) + local dk, dv = local dv + the update's, in the activation
// dtype.  One thread per element of k.
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_bwd_final(const T *__restrict__ k, BwdWs w, T *__restrict__ dk, T *__restrict__ dv,
            int64_t L, int N, int S, int64_t n)
{
    // four consecutive elements of one row per thread (d is a multiple of 4; the workspace
    // arrays are 256-byte aligned and the activations 16-byte aligned)
    const int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 4;
    if (i >= n) return;
    const int64_t row = i / D, a = i % D;
    const int64_t chain = row / L, t = row % L;
    const int s = (int)(t / N);
    const float4 ds = *reinterpret_cast<const float4 *>(w.dsk + i);
    const float4 zs = *reinterpret_cast<const float4 *>(w.dzs + (chain * S + s) * D + a);
    const float4 lk = *reinterpret_cast<const float4 *>(w.dk + i);
    const float4 lv = *reinterpret_cast<const float4 *>(w.dv + i);
    const float g[4] = {ds.x + zs.x, ds.y + zs.y, ds.z + zs.z, ds.w + zs.w};
    const float l4[4] = {lk.x, lk.y, lk.z, lk.w};
    const float v4[4] = {lv.x, lv.y, lv.z, lv.w};
    if constexpr (sizeof(T) == 2) {
        const uint2 kr = *reinterpret_cast<const uint2 *>(k + i);
        const float kx[4] = {__uint_as_float(kr.x << 16), __uint_as_float(kr.x & 0xffff0000u),
                             __uint_as_float(kr.y << 16), __uint_as_float(kr.y & 0xffff0000u)};
        float o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) o[u] = g[u] * sigma_grad(kx[u]) + l4[u];
        __nv_bfloat162 k01 = __floats2bfloat162_rn(o[0], o[1]), k23 = __floats2bfloat162_rn(o[2], o[3]);
        __nv_bfloat162 v01 = __floats2bfloat162_rn(v4[0], v4[1]), v23 = __floats2bfloat162_rn(v4[2], v4[3]);
        *reinterpret_cast<uint2 *>(dk + i) = make_uint2(*reinterpret_cast<uint32_t *>(&k01),
                                                        *reinterpret_cast<uint32_t *>(&k23));
        *reinterpret_cast<uint2 *>(dv + i) = make_uint2(*reinterpret_cast<uint32_t *>(&v01),
                                                        *reinterpret_cast<uint32_t *>(&v23));
    } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            st_f(dk + i + u, g[u] * sigma_grad(ld_f(k + i + u)) + l4[u]);
            st_f(dv + i + u, v4[u]);
        }
    }
}

// dbeta[h] = sum over batches, segments and row tiles of the partial sums (fixed order).
__global__ void __launch_bounds__(256)
k_bwd_beta(const float *part, float *dbeta, int B, int H, int S, int qtiles)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float t = 0.f;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < S * qtiles; ++i) t += part[((int64_t)b * H + h) * S * qtiles + i];
    dbeta[h] = t;
}

}  // namespace infini
