// CUDA-core (FFMA) kernels of the Infini-attention forward.
//
// These carry the fp32-activation path (exact fp32 products keep it inside the fp32
// tolerance, which tf32 tensor-core math would not) and every shape the tensor-core
// kernels do not specialise.  All arithmetic is fp32; inputs are fp32 or bf16.
//
// Equations: AI Wiki "Infini-Attention", "What happens inside the Infini-attention
// block?" (local causal softmax, sigma = ELU + 1 retrieval, sigmoid gate) and "How does
// the compressive memory work?" (linear / delta memory updates and the z update).
//
// Workspace convention shared with the host code: for chain c = b * Hkv + kvh and segment
// s, snapM[(c * S + s) * d * d ...] and snapZ[(c * S + s) * d ...] hold (M_{s-1}, z_{s-1}),
// the memory the segment reads.
//
// `valid` is the number of tokens the LAST segment of a launch really has (N when it is a
// full one; every earlier segment has N).  A final segment shorter than N runs with its
// rows past `valid` never read (they count as a zero key / value whose feature map is 0,
// not sigma(0)) and never written; the segment kernel runs such a segment alone, with N
// rounded up to 64.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace infini {

__device__ __forceinline__ float ld_f(const float *p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// sigma(x) = ELU(x) + 1 with alpha = 1.
__device__ __forceinline__ float feature_map(float x) { return x > 0.f ? x + 1.f : expf(x); }

// ---------------------------------------------------------------------------------------
// Linear rule, step 1: per (chain, segment) the increments dM_s = sigma(K_s)^T V_s and
// dz_s = sum_t sigma(K_s,t), written into the snapshot slot of that segment (the scan
// below turns the slots into exclusive prefix sums).  One CTA per (chain, segment).
// With `accumulate` set the increments are added to the slot instead (S = 1 and the slot
// is the memory itself: the in-place fold of one segment; each element has one owner).
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_linear_increments(const T *__restrict__ k, const T *__restrict__ v, float *__restrict__ snapM,
                    float *__restrict__ snapZ, int64_t L, int N, int S, int valid,
                    int accumulate = 0)
{
    constexpr int TK = 32, R = D / 16;
    __shared__ float sK[TK][D + 1];
    __shared__ float sV[TK][D + 1];
    const int64_t chain = blockIdx.x / S;
    const int s = blockIdx.x % S;
    const int vs = s == S - 1 ? valid : N;          // tokens of this segment
    const T *K = k + (chain * L + (int64_t)s * N) * D;
    const T *V = v + (chain * L + (int64_t)s * N) * D;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;

    float acc[R][R];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = 0.f;
    float zacc = 0.f;

    for (int t0 = 0; t0 < N; t0 += TK) {
        for (int i = tid; i < TK * D; i += 256) {
            const int t = i / D, c = i % D;
            const bool in = t0 + t < vs;
            sK[t][c] = in ? feature_map(ld_f(K + (int64_t)(t0 + t) * D + c)) : 0.f;
            sV[t][c] = in ? ld_f(V + (int64_t)(t0 + t) * D + c) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < TK; ++t) {
            float a[R], b[R];
#pragma unroll
            for (int i = 0; i < R; ++i) a[i] = sK[t][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < R; ++j) b[j] = sV[t][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < R; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (tid < D)
            for (int t = 0; t < TK; ++t) zacc += sK[t][tid];
        __syncthreads();
    }
    float *dst = snapM + (chain * S + s) * (int64_t)D * D;
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) {
            float *e = dst + (ty + 16 * i) * D + tx + 16 * j;
            *e = accumulate ? *e + acc[i][j] : acc[i][j];
        }
    if (tid < D) {
        float *e = snapZ + (chain * S + s) * D + tid;
        *e = accumulate ? *e + zacc : zacc;
    }
}

// ---------------------------------------------------------------------------------------
// z += sum_{t < valid} sigma(k_t) for every chain, in place (the delta rule's in-place fold
// writes M by column blocks and leaves z to this kernel, so that no CTA of the chain reads
// a z another CTA has already advanced).  One CTA per chain.
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
k_z_fold(const T *__restrict__ k, float *z, int64_t L, int valid)
{
    constexpr int PARTS = 256 / D;
    __shared__ float part[PARTS][D];
    const int64_t chain = blockIdx.x;
    const int f = threadIdx.x % D, p = threadIdx.x / D;
    const T *K = k + chain * L * D;
    float acc = 0.f;
    for (int t = p; t < valid; t += PARTS) acc += feature_map(ld_f(K + (int64_t)t * D + f));
    part[p][f] = acc;
    __syncthreads();
    if (threadIdx.x < D) {
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < PARTS; ++i) sum += part[i][f];
        z[chain * D + f] += sum;
    }
}

// ---------------------------------------------------------------------------------------
// Linear rule, step 2: exclusive prefix over segments, in place.  Slot s becomes
// M0 + sum_{j<s} dM_j (and the same for z); the inclusive total goes to M_out / z_out.
// One thread per state element; each thread reads its M0 element before writing the same
// element of M_out, so exact aliasing of M_out with M0 is safe.
// ---------------------------------------------------------------------------------------
// snapMb, when not NULL, receives bf16 copies of the M snapshots (the operand layout of
// the tensor-core segment kernel); the fp32 M snapshots are then not written back.
__global__ void __launch_bounds__(256)
k_linear_scan(float *__restrict__ snapM, float *__restrict__ snapZ,
              __nv_bfloat16 *__restrict__ snapMb, const float *M0, const float *z0,
              float *M_out, float *z_out, int S, int D, int64_t chains)
{
    const int64_t per = (int64_t)D * D + D;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= chains * per) return;
    const int64_t chain = idx / per;
    int64_t e = idx % per;
    if (e < (int64_t)D * D) {
        const int64_t o = chain * D * D + e;
        float run = M0 ? M0[o] : 0.f;
        float *p = snapM + chain * S * (int64_t)D * D + e;
        if (snapMb) {
            __nv_bfloat16 *pb = snapMb + chain * S * (int64_t)D * D + e;
            for (int s = 0; s < S; ++s) {
                const float x = p[(int64_t)s * D * D];
                pb[(int64_t)s * D * D] = __float2bfloat16_rn(run);
                run += x;
            }
        } else {
            for (int s = 0; s < S; ++s) {
                const float x = p[(int64_t)s * D * D];
                p[(int64_t)s * D * D] = run;
                run += x;
            }
        }
        M_out[o] = run;
    } else {
        e -= (int64_t)D * D;
        const int64_t o = chain * D + e;
        float run = z0 ? z0[o] : 0.f;
        float *p = snapZ + chain * S * (int64_t)D + e;
        for (int s = 0; s < S; ++s) {
            const float x = p[(int64_t)s * D];
            p[(int64_t)s * D] = run;
            run += x;
        }
        z_out[o] = run;
    }
}

// ---------------------------------------------------------------------------------------
// Delta rule, step 1: slot 0 of every chain <- (M0, z0) or zeros.  Done before the chain
// kernel so that kernel never reads M0 / z0 (which may alias M_out / z_out).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_state_init(const float *M0, const float *z0, float *__restrict__ snapM,
             float *__restrict__ snapZ, __nv_bfloat16 *__restrict__ snapMb, int S, int D,
             int64_t chains)
{
    const int64_t per = (int64_t)D * D + D;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= chains * per) return;
    const int64_t chain = idx / per;
    int64_t e = idx % per;
    if (e < (int64_t)D * D) {
        const float m = M0 ? M0[chain * D * D + e] : 0.f;
        snapM[chain * S * (int64_t)D * D + e] = m;
        if (snapMb) snapMb[chain * S * (int64_t)D * D + e] = __float2bfloat16_rn(m);
    } else {
        e -= (int64_t)D * D;
        snapZ[chain * S * (int64_t)D + e] = z0 ? z0[chain * D + e] : 0.f;
    }
}

// ---------------------------------------------------------------------------------------
// Delta rule, step 2: the sequential chain.  The update of value column e needs only
// column e of M_{s-1}, column e of V_s and the shared z_{s-1}, so each CTA owns CB columns
// of one chain's M (in shared memory, fp32) and walks all S segments; z is recomputed by
// every CTA of the chain (z_out NULL: z is not written).  Before segment s >= 1 the CTA publishes its columns of M_{s-1}
// into snapshot slot s (CTA 0 of the chain also publishes z).  Within a segment every
// token's prediction reads M_{s-1}: the increments are accumulated in registers and added
// after the whole segment.
// ---------------------------------------------------------------------------------------
template <typename T, int D, int CB>
__global__ void __launch_bounds__(256)
k_delta_chain(const T *__restrict__ k, const T *__restrict__ v, float *snapM,
              float *snapZ, __nv_bfloat16 *__restrict__ snapMb, float *M_out,
              float *z_out, int64_t L, int N, int S, int valid)
{
    constexpr int TK = 32, NBLK = D / CB, PER = D * CB / 256;
    static_assert(PER >= 1 && (D * CB) % 256 == 0, "column block too small");
    __shared__ float sM[D][CB];
    __shared__ float sz[D];
    __shared__ float sK[TK][D + 1];
    __shared__ float sV[TK][CB];
    __shared__ float sU[TK][CB];
    __shared__ float sden[TK];

    const int64_t chain = blockIdx.x / NBLK;
    const int cb = (blockIdx.x % NBLK) * CB;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    float *chainM = snapM + chain * S * (int64_t)D * D;
    float *chainZ = snapZ + chain * S * (int64_t)D;

    for (int i = tid; i < D * CB; i += 256) sM[i / CB][i % CB] = chainM[(i / CB) * D + cb + i % CB];
    for (int i = tid; i < D; i += 256) sz[i] = chainZ[i];
    __syncthreads();

    for (int s = 0; s < S; ++s) {
        if (s > 0) {
            if (snapMb) {
                __nv_bfloat16 *dst = snapMb + (chain * S + s) * (int64_t)D * D;
                for (int i = tid; i < D * CB; i += 256)
                    dst[(i / CB) * D + cb + i % CB] = __float2bfloat16_rn(sM[i / CB][i % CB]);
            } else {
                float *dst = chainM + (int64_t)s * D * D;
                for (int i = tid; i < D * CB; i += 256) dst[(i / CB) * D + cb + i % CB] = sM[i / CB][i % CB];
            }
            if (cb == 0)
                for (int i = tid; i < D; i += 256) chainZ[(int64_t)s * D + i] = sz[i];
        }
        const T *K = k + (chain * L + (int64_t)s * N) * D;
        const T *V = v + (chain * L + (int64_t)s * N) * D;
        const int vs = s == S - 1 ? valid : N;      // tokens of this segment
        float dm[PER];
#pragma unroll
        for (int p = 0; p < PER; ++p) dm[p] = 0.f;
        float dz = 0.f;

        for (int t0 = 0; t0 < N; t0 += TK) {
            for (int i = tid; i < TK * D; i += 256) {
                const int t = i / D, c = i % D;
                sK[t][c] = t0 + t < vs ? feature_map(ld_f(K + (int64_t)(t0 + t) * D + c)) : 0.f;
            }
            for (int i = tid; i < TK * CB; i += 256) {
                const int t = i / CB, e = i % CB;
                sV[t][e] = t0 + t < vs ? ld_f(V + (int64_t)(t0 + t) * D + cb + e) : 0.f;
            }
            __syncthreads();
            // den_t = sigma(k_t) . z_{s-1}: one warp per token
            for (int t = warp; t < TK; t += 8) {
                float part = 0.f;
                for (int c = lane; c < D; c += 32) part = fmaf(sK[t][c], sz[c], part);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) sden[t] = part;
            }
            __syncthreads();
            // U = V - sigma(K) M_{s-1} / den  (0 prediction where den == 0)
            for (int i = tid; i < TK * CB; i += 256) {
                const int t = i / CB, e = i % CB;
                float r = 0.f;
#pragma unroll 8
                for (int c = 0; c < D; ++c) r = fmaf(sK[t][c], sM[c][e], r);
                const float den = sden[t];
                sU[t][e] = sV[t][e] - (den == 0.f ? 0.f : r / den);
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
            if (tid < D)
                for (int t = 0; t < TK; ++t) dz += sK[t][tid];
            __syncthreads();
        }
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            const int i = tid + 256 * p;
            sM[i / CB][i % CB] += dm[p];
        }
        if (tid < D) sz[tid] += dz;
        __syncthreads();
    }
    for (int i = tid; i < D * CB; i += 256) M_out[chain * D * D + (i / CB) * D + cb + i % CB] = sM[i / CB][i % CB];
    if (cb == 0 && z_out)
        for (int i = tid; i < D; i += 256) z_out[chain * D + i] = sz[i];
}

// ---------------------------------------------------------------------------------------
// Segment kernel (CUDA cores): one CTA per 64 query rows of one (b, h, segment).
// Local causal attention with an online softmax over 64-key tiles of the same segment up
// to the diagonal, then the retrieval sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}) from the
// snapshot slot, then the gate and the store.
// ---------------------------------------------------------------------------------------
template <int D>
struct SimtSegSmem {
    static constexpr int BQ = 64, BK = 64;
    static constexpr int floats = BQ * (D + 1) + BK * (D + 1) + BK * D + BQ * (BK + 1);
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
k_segment_simt(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
               const float *__restrict__ beta, const float *__restrict__ snapM,
               const float *__restrict__ snapZ, T *__restrict__ out, int64_t L, int N, int S,
               int H, int Hkv, int valid)
{
    constexpr int BQ = 64, BK = 64, RJ = D / 16;
    extern __shared__ float smem[];
    float *sQ = smem;                    // [BQ][D+1]
    float *sK = sQ + BQ * (D + 1);       // [BK][D+1]
    float *sV = sK + BK * (D + 1);       // [BK][D]
    float *sP = sV + BK * D;             // [BQ][BK+1]

    const int qtiles = N / BQ;
    int64_t bid = blockIdx.x;
    const int qt = (int)(bid % qtiles); bid /= qtiles;
    const int s = (int)(bid % S); bid /= S;
    const int64_t bh = bid;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int kvh = h / (H / Hkv);
    const int64_t chain = b * Hkv + kvh;
    const int64_t tok0 = (int64_t)s * N + (int64_t)qt * BQ;
    const T *Q = q + (bh * L + tok0) * D;
    const T *Kseg = k + (chain * L + (int64_t)s * N) * D;
    const T *Vseg = v + (chain * L + (int64_t)s * N) * D;

    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int q0 = qt * BQ;                 // first query row within the segment
    for (int i = tid; i < BQ * D; i += 256)
        sQ[(i / D) * (D + 1) + i % D] = q0 + i / D < valid ? ld_f(Q + i) : 0.f;

    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;   // softmax scale * log2(e)
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
                if (kt == qt && c > r) x = -INFINITY;
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

    // ---- retrieval from M_{s-1}, z_{s-1} ----
    __syncthreads();
    for (int i = tid; i < BQ * D; i += 256) {
        float *p = sQ + (i / D) * (D + 1) + i % D;
        *p = feature_map(*p);
    }
    const float *Ms = snapM + (chain * S + s) * (int64_t)D * D;
    const float *zs = snapZ + (chain * S + s) * (int64_t)D;
    float *sZ = sP;                       // z_{s-1}, D floats
    for (int i = tid; i < D; i += 256) sZ[i] = zs[i];
    __syncthreads();
    float den[4], num[4][RJ];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a = 0.f;
        for (int c = 0; c < D; ++c) a = fmaf(sQ[(ty + 16 * i) * (D + 1) + c], sZ[c], a);
        den[i] = a;
#pragma unroll
        for (int j = 0; j < RJ; ++j) num[i][j] = 0.f;
    }
    float *sMc = sK;                      // 32 rows of M at a time: [32][D]
    for (int kc = 0; kc < D; kc += 32) {
        __syncthreads();
        for (int i = tid; i < 32 * D; i += 256) sMc[i] = Ms[(int64_t)kc * D + i];
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < 32; ++kk) {
            float mm[RJ];
#pragma unroll
            for (int j = 0; j < RJ; ++j) mm[j] = sMc[kk * D + tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = sQ[(ty + 16 * i) * (D + 1) + kc + kk];
#pragma unroll
                for (int j = 0; j < RJ; ++j) num[i][j] = fmaf(a, mm[j], num[i][j]);
            }
        }
    }
    const float g = 1.f / (1.f + expf(-beta[h]));
    T *O = out + (bh * L + tok0) * D;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
        if (q0 + r >= valid) continue;
        const float inv_l = 1.f / l[i];
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
            const float amem = den[i] == 0.f ? 0.f : num[i][j] / den[i];
            st_f(O + (int64_t)r * D + tx + 16 * j, g * amem + (1.f - g) * (o[i][j] * inv_l));
        }
    }
}

}  // namespace infini
