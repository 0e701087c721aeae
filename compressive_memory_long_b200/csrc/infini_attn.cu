// Host side of the C ABI declared in include/infini_attn.h: argument checks, workspace,
// kernel selection and launches.  No torch types cross this boundary.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "infini_attn.h"
#include "simt_kernels.cuh"
#include "tc_segment.cuh"
#include "tc_segment_p.cuh"
#include "tc_backward.cuh"
#include "tc_memory.cuh"
#include "tc_small.cuh"
#include "tc_pieces.cuh"
#include "decode.cuh"
#include "backward.cuh"

#include <cudaTypedefs.h>

// Workspace of infini_attn_fwd_noalloc: a file-scope device array used instead of a
// per-call allocation.  Every GPU that loads the library holds it until the process exits.
// In host code the name is only a host-side stand-in for the symbol, never a device
// address: the address comes from cudaGetSymbolAddress, looked up once per device with that
// device current (noalloc_scratch_address below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[INFINI_NOALLOC_SCRATCH_BYTES];

namespace infini {
namespace {

// L is the row count of every head (the row stride of q, k, v, out); S = floor(L / N) full
// segments cover the first Lf = S * N rows and T = L - Lf rows (0 <= T < N) form a final,
// shorter segment.
struct Problem {
    int64_t B, H, Hkv, L, N, d, S, Lf, T;
    int rule;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a+na) and [b, b+nb) overlap without being the same range
bool partial_overlap(const void *a, int64_t na, const void *b, int64_t nb)
{
    if (!a || !b) return false;
    const uintptr_t a0 = (uintptr_t)a, a1 = a0 + (uintptr_t)na;
    const uintptr_t b0 = (uintptr_t)b, b1 = b0 + (uintptr_t)nb;
    if (a0 == b0 && na == nb) return false;
    return a0 < b1 && b0 < a1;
}

bool ranges_overlap(const void *a, int64_t na, const void *b, int64_t nb)
{
    if (!a || !b) return false;
    const uintptr_t a0 = (uintptr_t)a, a1 = a0 + (uintptr_t)na;
    const uintptr_t b0 = (uintptr_t)b, b1 = b0 + (uintptr_t)nb;
    return a0 < b1 && b0 < a1;
}

int check_args(const void *q, const void *k, const void *v, const float *beta, const float *M0,
               const float *z0, const void *out, const float *M_out, const float *z_out,
               int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N, int64_t d, int rule,
               int64_t esize, Problem *pb, bool out_checked = true)
{
    if (!q || !k || !v || !beta || !out || !M_out || !z_out) return INFINI_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || Hkv <= 0 || L <= 0 || N <= 0 || d <= 0) return INFINI_ERR_INVALID_ARG;
    if (H % Hkv != 0) return INFINI_ERR_INVALID_ARG;
    if (rule != INFINI_UPDATE_LINEAR && rule != INFINI_UPDATE_DELTA) return INFINI_ERR_INVALID_ARG;
    // keep every element count far inside int64 and every grid inside 2^31 CTAs
    if (B > (1 << 20) || H > (1 << 16) || L > ((int64_t)1 << 34) ||
        B * H * L > ((int64_t)1 << 40) || B * H * (L / 128) > ((int64_t)1 << 30))
        return INFINI_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, beta, M0, z0, out, M_out, z_out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return INFINI_ERR_INVALID_ARG;
    const int64_t mbytes = B * Hkv * d * d * 4, zbytes = B * Hkv * d * 4;
    if (partial_overlap(M0, mbytes, M_out, mbytes) || partial_overlap(z0, zbytes, z_out, zbytes))
        return INFINI_ERR_INVALID_ARG;
    const int64_t obytes = B * H * L * d * esize, kvbytes = B * Hkv * L * d * esize;
    if (out_checked &&
        (ranges_overlap(out, obytes, q, obytes) || ranges_overlap(out, obytes, k, kvbytes) ||
         ranges_overlap(out, obytes, v, kvbytes) || ranges_overlap(out, obytes, M_out, mbytes) ||
         ranges_overlap(out, obytes, z_out, zbytes)))
        return INFINI_ERR_INVALID_ARG;
    if (ranges_overlap(M_out, mbytes, z_out, zbytes)) return INFINI_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 128) return INFINI_ERR_UNSUPPORTED;
    if (N % 64 != 0) return INFINI_ERR_UNSUPPORTED;
    pb->B = B; pb->H = H; pb->Hkv = Hkv; pb->L = L; pb->N = N; pb->d = d; pb->S = L / N;
    pb->Lf = pb->S * N; pb->T = L - pb->Lf;
    pb->rule = rule;
    return INFINI_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).  Setting the
// same value twice is harmless, so racing first calls need no lock.
template <auto Kernel>
bool opt_in_smem(size_t bytes)
{
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = 1ull << (dev & 63);
    if (done_mask.load(std::memory_order_relaxed) & bit) return true;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return false;
    done_mask.fetch_or(bit);
    return true;
}

// SMs of the current device (148 on a B200 if the query fails).
int sm_count()
{
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        sms = 148;
    }
    return sms;
}

// ---- opt-in launch tracing: a pair of CUDA events on the launch stream around every
// kernel this library enqueues, read back (and cleared) by infini_attn_trace_report ----
namespace trace {
struct Rec {
    const char *name;
    cudaEvent_t a, b;
};
std::mutex mu;
std::vector<Rec> recs;                  // launches not yet folded into the table
std::vector<std::string> names;         // accumulated table: kernel, launches, device ms
std::vector<int64_t> counts;
std::vector<double> ms;
std::vector<cudaEvent_t> pool;          // events ready for reuse (each belongs to one device)
std::vector<int> pool_dev;
bool failed = false;
std::atomic<int> enabled{0};

// An event of the current device from the pool, or a new one.
bool take_event(cudaEvent_t *e)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    {
        std::lock_guard<std::mutex> g(mu);
        for (size_t i = pool.size(); i-- > 0;)
            if (pool_dev[i] == dev) {
                *e = pool[i];
                pool.erase(pool.begin() + i);
                pool_dev.erase(pool_dev.begin() + i);
                return true;
            }
    }
    return cudaEventCreate(e) == cudaSuccess;
}

void give_event(cudaEvent_t e)
{
    int dev = 0;
    cudaGetDevice(&dev);
    pool.push_back(e);          // callers hold mu
    pool_dev.push_back(dev);
}

struct Scope {
    Rec r{};
    bool on;
    cudaStream_t st;
    Scope(const char *name, cudaStream_t s) : on(enabled.load() != 0), st(s)
    {
        if (!on) return;
        r.name = name;
        if (!take_event(&r.a) || !take_event(&r.b)) {
            on = false;
            return;
        }
        cudaEventRecord(r.a, st);
    }
    ~Scope()
    {
        if (!on) return;
        cudaEventRecord(r.b, st);
        std::lock_guard<std::mutex> g(mu);
        recs.push_back(r);
    }
};
}  // namespace trace

#define TRACED(name, st) trace::Scope trace_scope(name, st)

// ---- TMA tensor maps (driver entry point fetched through the runtime: no libcuda link) ----
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor [d2][d1][d0] (d0 contiguous) read as boxes of box1 rows x box0 columns.
// With the 128-byte swizzle box0 is 64 (128 bytes) and every box starts at a column multiple
// of 64; unswizzled boxes start at column multiples of 8 (16 bytes).
bool make_map_bf16_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t box1, uint32_t box0 = 64, bool swizzle128 = true)
{
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core path covers bf16 activations, d in {64, 128}, N % 128 == 0 or N = 64
// (two 64-token segments per 128-row tile).
template <typename T>
bool use_tc(const Problem &p)
{
    return sizeof(T) == 2 && (p.d == 64 || p.d == 128) && (p.N % 128 == 0 || p.N == 64);
}

// One launch for 64-token segments under the additive rule (bf16, d = 64): whole 128-token
// units only, so never a problem whose last segment is short (L < Lf once effective() has
// made a short tail one more segment).
template <typename T>
bool use_small_fused(const Problem &p)
{
    return sizeof(T) == 2 && p.d == 64 && p.N == 64 && p.rule == INFINI_UPDATE_LINEAR &&
           p.Lf % 128 == 0 && p.L >= p.Lf;
}

// Long heads (16 units of 128 tokens or more) go to the persistent piece kernel.
bool use_pieces(const Problem &p) { return p.Lf / 128 >= 16; }

// Workspace of one call.  CUDA-core path: fp32 snapshots (M_{s-1}, z_{s-1}) of every
// segment.  Tensor-core path: z_{s-1} and dz_s (fp32), the bf16 snapshots M_{s-1} the
// segment kernel reads, the increments B_s (fp32) and, for the delta rule, A_s in two bf16
// parts.  A final short segment counts as a segment.  The fused 64-token paths size their
// own (much smaller) workspace.
int64_t simt_workspace_bytes(int64_t units, int64_t d) { return units * (d * d + d) * 4 + 256; }

int64_t tc_workspace_bytes(int64_t units, int64_t d, bool delta)
{
    return units * (2 * d * 4 + d * d * 2 + d * d * 4 + (delta ? 2 * d * d * 2 : 0)) + 256;
}

// An upper bound over every path (the exported figure).
int64_t workspace_bytes(int64_t B, int64_t Hkv, int64_t L, int64_t N, int64_t d)
{
    const int64_t units = B * Hkv * ((L + N - 1) / N);
    return std::max(simt_workspace_bytes(units, d), tc_workspace_bytes(units, d, true));
}

// Pointers into one call's workspace.
struct Workspace {
    void *raw = nullptr;
    float *snapM = nullptr, *snapZ = nullptr;          // CUDA-core path
    float *dz = nullptr, *Bs = nullptr;                // tensor-core path (+ snapZ)
    __nv_bfloat16 *snapMb = nullptr, *Ahi = nullptr, *Alo = nullptr;
};

Workspace carve_workspace(void *raw, int64_t units, int64_t d, bool tc_path)
{
    Workspace w;
    w.raw = raw;
    if (!raw) return w;
    char *c = static_cast<char *>(raw);
    if (!tc_path) {
        w.snapM = reinterpret_cast<float *>(c);
        w.snapZ = w.snapM + units * d * d;
        return w;
    }
    w.snapZ = reinterpret_cast<float *>(c);
    w.dz = w.snapZ + units * d;
    w.Bs = w.dz + units * d;
    w.snapMb = reinterpret_cast<__nv_bfloat16 *>(w.Bs + units * d * d);
    w.Ahi = w.snapMb + units * d * d;
    w.Alo = w.Ahi + units * d * d;
    return w;
}

// The memory path of the tensor-core forward: z prefix, per-segment increments on the
// tensor cores, then the recurrence (delta) or the running sum (linear).  Leaves the
// snapshots (z_{s-1} fp32, M_{s-1} bf16) for the segment kernel, and M_out / z_out.
template <int D>
int launch_memory_tc(const Problem &p, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                     const float *M0, const float *z0, const Workspace &ws, float *M_out,
                     float *z_out, cudaStream_t st, float *snapMf = nullptr)
{
    const int64_t chains = p.B * p.Hkv, units = chains * p.S;
    const int S = (int)p.S, N = (int)p.N;
    const bool delta = p.rule == INFINI_UPDATE_DELTA;
    // the delta rule's increments need z_{s-1}: sum sigma(K) per segment first; the additive
    // rule's increments kernel sums it itself on the tensor cores and the scan follows
    if (delta) {
        TRACED("z_sum", st);
        tc::k_zsum<D><<<(unsigned)units, 256, 0, st>>>(k, ws.dz, p.L, N, S);
    }
    auto z_scan = [&]() {
        TRACED("z_scan", st);
        tc::k_zscan<D><<<(unsigned)chains, D * 8, 0, st>>>(ws.dz, z0, ws.snapZ, z_out, S);
    };
    if (delta) z_scan();
    CUtensorMap mk, mv;
    if (!make_map_bf16_3d(&mk, k, D, p.L, chains, 64) || !make_map_bf16_3d(&mv, v, D, p.L, chains, 64))
        return INFINI_ERR_CUDA;
    // persistent: one CTA per SM (or per item when there are fewer)
    tc::IncrArgs ia{ws.snapZ, ws.Bs, ws.Ahi, ws.Alo, ws.dz, p.L, N, S, (int)units};
    const unsigned igrid = (unsigned)std::min<int64_t>(units, sm_count());
    if (delta) {
        using C = tc::IncrCfg<D, true>;
        if (!opt_in_smem<tc::k_mem_incr<D, true>>(C::ALLOC)) return INFINI_ERR_CUDA;
        TRACED("mem_increments", st);
        tc::k_mem_incr<D, true><<<igrid, C::THREADS, C::ALLOC, st>>>(mk, mv, ia);
    } else {
        using C = tc::IncrCfg<D, false>;
        if (!opt_in_smem<tc::k_mem_incr<D, false>>(C::ALLOC)) return INFINI_ERR_CUDA;
        TRACED("mem_increments", st);
        tc::k_mem_incr<D, false><<<igrid, C::THREADS, C::ALLOC, st>>>(mk, mv, ia);
    }
    if (!delta) {
        z_scan();
        const int64_t n4 = chains * D * D / 4;
        TRACED("mem_prefix", st);
        // many segments: 8 chunks per element walked side by side; few: one walk
        if (S >= 64)
            tc::k_mem_prefix<D, 8><<<(unsigned)((n4 + 31) / 32), 256, 0, st>>>(ws.Bs, M0, ws.snapMb, M_out,
                                                                            S, chains, snapMf);
        else
            tc::k_mem_prefix<D, 1><<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(ws.Bs, M0, ws.snapMb, M_out,
                                                                              S, chains, snapMf);
        return INFINI_OK;
    }
    using MC = tc::MChainCfg<D>;
    CUtensorMap mah, mal;
    if (!make_map_bf16_3d(&mah, ws.Ahi, D, D, units, D) ||
        !make_map_bf16_3d(&mal, ws.Alo, D, D, units, D))
        return INFINI_ERR_CUDA;
    if (!opt_in_smem<tc::k_mem_chain<D>>(MC::ALLOC)) return INFINI_ERR_CUDA;
    tc::MChainArgs ca{M0, ws.Bs, ws.snapMb, snapMf, M_out, S, 0};
    TRACED("mem_chain", st);
    tc::k_mem_chain<D><<<(unsigned)(chains * (D / MC::CB)), MC::THREADS, MC::ALLOC, st>>>(mah, mal, ca);
    return INFINI_OK;
}

// The two-tile kernel redistributes registers with setmaxnreg; its split assumes the
// register count per thread it was compiled with.  Checked once per kernel: a mismatch
// would leave the growing warpgroups waiting forever, so the one-tile kernel runs instead.
template <int D>
bool segp_registers_match()
{
    static const bool ok = [] {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, tc::k_segment_tcp<D>) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        return fa.numRegs == tc::SegPCfg<D>::REGS;
    }();
    return ok;
}

template <int D>
int launch_segment_tc(const Problem &p, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                      const __nv_bfloat16 *v, const float *beta, const __nv_bfloat16 *snapMb,
                      const float *snapZ, __nv_bfloat16 *out, cudaStream_t st)
{
    using C = tc::SegCfg<D>;
    CUtensorMap mq, mk, mv, mm;
    if (!make_map_bf16_3d(&mq, q, D, p.L, p.B * p.H, 128) ||
        !make_map_bf16_3d(&mk, k, D, p.L, p.B * p.Hkv, 128) ||
        !make_map_bf16_3d(&mv, v, D, p.L, p.B * p.Hkv, 128) ||
        !make_map_bf16_3d(&mm, snapMb, D, D, p.B * p.Hkv * p.S, D))
        return INFINI_ERR_CUDA;
    tc::SegArgs a{beta, snapZ, out, p.L, (int)p.N, (int)p.S, (int)p.H, (int)p.Hkv};
    if (p.N % 256 == 0 && segp_registers_match<D>()) {
        // persistent, two query tiles per work item: one CTA per SM over balanced units
        using CP = tc::SegPCfg<D>;
        CUtensorMap mo;
        if (!make_map_bf16_3d(&mo, out, D, p.L, p.B * p.H, 128)) return INFINI_ERR_CUDA;
        if (!opt_in_smem<tc::k_segment_tcp<D>>(CP::ALLOC)) return INFINI_ERR_CUDA;
        const int64_t units = p.B * p.H * p.S * ((p.N / 256 + 1) / 2);
        if (units >= (int64_t)1 << 31) return INFINI_ERR_UNSUPPORTED;   // beyond any device memory
        const int64_t ctas = units < sm_count() ? units : sm_count();
        TRACED("segment_tc", st);
        tc::k_segment_tcp<D><<<(unsigned)ctas, CP::THREADS, CP::ALLOC, st>>>(mq, mk, mv, mm, mo, a,
                                                                              (uint32_t)units);
        return INFINI_OK;
    }
    if (!opt_in_smem<tc::k_segment_tc<D>>(C::ALLOC)) return INFINI_ERR_CUDA;
    // N = 64: one CTA per pair of consecutive segments
    const int64_t ctas = p.N == 64 ? p.B * p.H * ((p.S + 1) / 2) : p.B * p.H * p.S * (p.N / 128);
    TRACED("segment_tc", st);
    tc::k_segment_tc<D><<<(unsigned)ctas, 256, C::ALLOC, st>>>(mq, mk, mv, mm, a);
    return INFINI_OK;
}

int64_t small_workspace_bytes(const Problem &p)
{
    const int64_t chains = p.B * p.H, units = chains * (p.Lf / 128);
    const int64_t head = ((64 + chains + units) * 4 + 255) / 256 * 256;
    return head + 2 * units * tc::SmallCfg::STATE * 4;
}

int launch_small_fused(const Problem &p, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                       const __nv_bfloat16 *v, const float *beta, const float *M0,
                       const float *z0, __nv_bfloat16 *out, float *M_out, float *z_out,
                       void *ws, cudaStream_t st)
{
    if (p.L < p.Lf || p.Lf % 128 != 0) return INFINI_ERR_UNSUPPORTED;   // whole 128-token units
    using C = tc::SmallCfg;
    const int64_t chains = p.B * p.H, U = p.Lf / 128, units = chains * U;   // query-head chains
    // workspace: ticket, per-head M0 reader counts, flags (all zeroed here), then the
    // published aggregates / prefixes
    int *ticket = static_cast<int *>(ws);
    int *m0_done = ticket + 64;
    int *flags = m0_done + chains;
    const size_t ints = 64 + chains + units;
    const size_t head = (ints * 4 + 255) / 256 * 256;
    float *agg = reinterpret_cast<float *>(static_cast<char *>(ws) + head);
    float *incl = agg + units * C::STATE;
    if (cudaMemsetAsync(ws, 0, ints * 4, st) != cudaSuccess) return INFINI_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    if (!make_map_bf16_3d(&mq, q, C::D, p.L, p.B * p.H, 128) ||
        !make_map_bf16_3d(&mk, k, C::D, p.L, p.B * p.Hkv, 128) ||
        !make_map_bf16_3d(&mv, v, C::D, p.L, p.B * p.Hkv, 128))
        return INFINI_ERR_CUDA;
    if (!opt_in_smem<tc::k_small_linear_fused>(C::ALLOC)) return INFINI_ERR_CUDA;
    // few units per head: each sums its predecessors' aggregates directly
    const int direct = U <= 64 ? 1 : 0;
    const int in_place = ((M0 && M0 == M_out) || (z0 && z0 == z_out)) ? 1 : 0;
    tc::SmallArgs a{beta, M0, z0, out, M_out, z_out, ticket, m0_done, flags, agg, incl,
                    p.L, (int)U, (int)p.H, (int)p.Hkv, (int)chains, direct, in_place};
    TRACED("small_fused", st);
    tc::k_small_linear_fused<<<(unsigned)units, 256, C::ALLOC, st>>>(mq, mk, mv, a);
    return INFINI_OK;
}


// Long heads of 64-token segments: the persistent piece kernel.  Units per piece: about four
// pieces per CTA across the grid, at most PieceCfg::MAX_UNITS.
struct PiecePlan {
    int64_t chains, U, UP, P, total;
};

PiecePlan piece_plan(const Problem &p)
{
    PiecePlan pl;
    pl.chains = p.B * p.H;
    pl.U = p.Lf / 128;
    const int64_t target = 4 * (int64_t)sm_count();
    int64_t up = (pl.chains * pl.U) / target;
    up = up < 1 ? 1 : (up > tc::PieceCfg::MAX_UNITS ? tc::PieceCfg::MAX_UNITS : up);
    pl.UP = up;
    pl.P = (pl.U + up - 1) / up;
    pl.total = pl.chains * pl.P;
    return pl;
}

// workspace of the piece kernel: ticket and flags (zeroed per call), then the published
// aggregate and inclusive prefix of every piece
int64_t pieces_workspace_bytes(const Problem &p)
{
    const PiecePlan pl = piece_plan(p);
    const int64_t head = ((64 + pl.total) * 4 + 255) / 256 * 256;
    return head + 2 * pl.total * tc::PieceCfg::STATE * 4;
}

int launch_pieces(const Problem &p, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                  const __nv_bfloat16 *v, const float *beta, const float *M0, const float *z0,
                  __nv_bfloat16 *out, float *M_out, float *z_out, void *ws, cudaStream_t st)
{
    if (p.L < p.Lf || p.Lf % 128 != 0) return INFINI_ERR_UNSUPPORTED;   // whole 128-token units
    using C = tc::PieceCfg;
    const PiecePlan pl = piece_plan(p);
    int *ticket = static_cast<int *>(ws);
    int *flags = ticket + 64;
    const size_t ints = 64 + pl.total;
    const size_t head = (ints * 4 + 255) / 256 * 256;
    float *agg = reinterpret_cast<float *>(static_cast<char *>(ws) + head);
    float *incl = agg + pl.total * C::STATE;
    if (cudaMemsetAsync(ws, 0, ints * 4, st) != cudaSuccess) return INFINI_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    if (!make_map_bf16_3d(&mq, q, C::D, p.L, p.B * p.H, 128) ||
        !make_map_bf16_3d(&mk, k, C::D, p.L, p.B * p.Hkv, 128) ||
        !make_map_bf16_3d(&mv, v, C::D, p.L, p.B * p.Hkv, 128))
        return INFINI_ERR_CUDA;
    if (!opt_in_smem<tc::k_small_pieces>(C::ALLOC)) return INFINI_ERR_CUDA;
    tc::PieceArgs a{beta, M0, z0, out, M_out, z_out, ticket, flags, agg, incl, p.L,
                    (int)pl.U, (int)pl.UP, (int)pl.P, (int)p.H, (int)p.Hkv, (int)pl.chains,
                    (int)pl.total};
    const int64_t sms = sm_count();
    const int64_t grid = pl.total < sms ? pl.total : sms;
    TRACED("small_pieces", st);
    tc::k_small_pieces<<<(unsigned)grid, C::THREADS, C::ALLOC, st>>>(mq, mk, mv, a);
    return INFINI_OK;
}

// outputs = false: the memory chain only (M_out, z_out), no segment kernel.
template <typename T, int D>
int launch_all(const Problem &p, const T *q, const T *k, const T *v, const float *beta,
               const float *M0, const float *z0, T *out, float *M_out, float *z_out,
               const Workspace &ws, cudaStream_t st, bool outputs = true)
{
    if constexpr (sizeof(T) == 2 && D == 64) {
        // grouped query heads with the state updated in place take the general path: a head
        // of the group could still be reading M0 / z0 when the group's writer replaces them
        const bool group_in_place = p.H != p.Hkv && ((M0 && M0 == M_out) || (z0 && z0 == z_out));
        if (outputs && use_small_fused<T>(p) && !group_in_place) {
            const int rc = use_pieces(p)
                ? launch_pieces(p, q, k, v, beta, M0, z0, out, M_out, z_out, ws.raw, st)
                : launch_small_fused(p, q, k, v, beta, M0, z0, out, M_out, z_out, ws.raw, st);
            if (rc != INFINI_OK) return rc;
            return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
        }
    }
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (ws.snapMb) {       // the tensor-core path
            int rc = launch_memory_tc<D>(p, k, v, M0, z0, ws, M_out, z_out, st);
            if (rc != INFINI_OK) return rc;
            if (outputs) {
                rc = launch_segment_tc<D>(p, q, k, v, beta, ws.snapMb, ws.snapZ, out, st);
                if (rc != INFINI_OK) return rc;
            }
            return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
        }
    }
    const int64_t chains = p.B * p.Hkv;
    const int S = (int)p.S, N = (int)p.N;
    const int64_t per = (int64_t)D * D + D;
    const unsigned state_grid = (unsigned)((chains * per + 255) / 256);
    float *snapM = ws.snapM, *snapZ = ws.snapZ;
    if (p.rule == INFINI_UPDATE_LINEAR) {
        {
            TRACED("linear_increments", st);
            k_linear_increments<T, D><<<(unsigned)(chains * S), 256, 0, st>>>(k, v, snapM, snapZ,
                                                                             p.L, N, S, N);
        }
        {
            TRACED("linear_scan", st);
            k_linear_scan<<<state_grid, 256, 0, st>>>(snapM, snapZ, nullptr, M0, z0, M_out, z_out,
                                                      S, D, chains);
        }
    } else {
        constexpr int CB = 16;
        {
            TRACED("state_init", st);
            k_state_init<<<state_grid, 256, 0, st>>>(M0, z0, snapM, snapZ, nullptr, S, D, chains);
        }
        TRACED("delta_chain", st);
        k_delta_chain<T, D, CB><<<(unsigned)(chains * (D / CB)), 256, 0, st>>>(
            k, v, snapM, snapZ, nullptr, M_out, z_out, p.L, N, S, N);
    }
    if (!outputs) return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
    const size_t smem = SimtSegSmem<D>::bytes;
    if (!opt_in_smem<k_segment_simt<T, D>>(smem)) return INFINI_ERR_CUDA;
    const int64_t ctas = p.B * p.H * p.S * (p.N / 64);
    {
        TRACED("segment_simt", st);
        k_segment_simt<T, D><<<(unsigned)ctas, 256, smem, st>>>(q, k, v, beta, snapM, snapZ, out,
                                                               p.L, N, S, (int)p.H, (int)p.Hkv, N);
    }
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// Fold the first n rows (stride L rows per chain) of k, v into (M, z), in place, with the
// CUDA-core state kernels run as one segment of n tokens (N rounded up to 64; rows past n
// are never read).  Linear: the increments are added into M and z by their owners.
// Delta: each CTA reads its column block of M and all of z, and writes back only its
// columns; z advances in a second kernel once every block has read it.  No workspace.
template <typename T, int D>
void launch_fold_inplace(const T *k, const T *v, int64_t L, int64_t n, float *M, float *z,
                         int64_t chains, int rule, cudaStream_t st)
{
    if (n <= 0) return;
    const int Np = (int)((n + 63) / 64 * 64);
    if (rule == INFINI_UPDATE_LINEAR) {
        TRACED("fold_linear", st);
        k_linear_increments<T, D><<<(unsigned)chains, 256, 0, st>>>(k, v, M, z, L, Np, 1, (int)n, 1);
        return;
    }
    {
        TRACED("fold_delta_chain", st);
        k_delta_chain<T, D, 16><<<(unsigned)(chains * (D / 16)), 256, 0, st>>>(
            k, v, M, z, nullptr, M, nullptr, L, Np, 1, (int)n);
    }
    TRACED("fold_z", st);
    k_z_fold<T, D><<<(unsigned)chains, 256, 0, st>>>(k, z, L, (int)n);
}

// The final short segment (T rows after the S full segments, 0 < T < N).  The state
// before it is in (M_out, z_out): the full segments left it there, or, without full
// segments, it is copied from (M0, z0) (zeros when NULL).  The CUDA-core segment kernel
// computes its outputs from that state (N rounded up to 64, valid = T); then the tail is
// folded into (M_out, z_out) in place.
template <typename T, int D>
int launch_tail(const Problem &p, const T *q, const T *k, const T *v, const float *beta,
                const float *M0, const float *z0, T *out, float *M_out, float *z_out,
                cudaStream_t st, bool outputs = true)
{
    const int64_t chains = p.B * p.Hkv, off = p.Lf * D;
    const int Tn = (int)p.T, Np = (Tn + 63) / 64 * 64;
    if (p.S == 0) {
        const size_t mb = (size_t)chains * D * D * 4, zb = (size_t)chains * D * 4;
        if (M0 != M_out &&
            (M0 ? cudaMemcpyAsync(M_out, M0, mb, cudaMemcpyDeviceToDevice, st)
                : cudaMemsetAsync(M_out, 0, mb, st)) != cudaSuccess)
            return INFINI_ERR_CUDA;
        if (z0 != z_out &&
            (z0 ? cudaMemcpyAsync(z_out, z0, zb, cudaMemcpyDeviceToDevice, st)
                : cudaMemsetAsync(z_out, 0, zb, st)) != cudaSuccess)
            return INFINI_ERR_CUDA;
    }
    const size_t smem = SimtSegSmem<D>::bytes;
    if (outputs && !opt_in_smem<k_segment_simt<T, D>>(smem)) return INFINI_ERR_CUDA;
    if (outputs) {
        TRACED("tail_segment", st);
        k_segment_simt<T, D><<<(unsigned)(p.B * p.H * (Np / 64)), 256, smem, st>>>(
            q + off, k + off, v + off, beta, M_out, z_out, out + off, p.L, Np, 1, (int)p.H,
            (int)p.Hkv, Tn);
    }
    launch_fold_inplace<T, D>(k + off, v + off, p.L, Tn, M_out, z_out, chains, p.rule, st);
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

// The problem the kernels run.  On the tensor-core path a final short segment is simply
// one more segment: TMA fills its rows past L with zeros, the memory kernels leave those
// rows out of the update (zero sigma(K)), and the segment kernel neither computes tiles
// that start past L nor stores rows past L.  Elsewhere, and after the fused 64-token
// kernels (which take whole 128-token units only), the CUDA-core tail follows the full
// segments.
template <typename T>
Problem effective(const Problem &p)
{
    Problem e = p;
    if (p.T > 0 && use_tc<T>(p) && !use_small_fused<T>(p)) {
        e.S = p.S + 1;
        e.Lf = e.S * p.N;
        e.T = 0;
    }
    return e;
}

// The full segments, then the final short one (if any).
template <typename T, int D>
int launch_forward(const Problem &p, const T *q, const T *k, const T *v, const float *beta,
                   const float *M0, const float *z0, T *out, float *M_out, float *z_out,
                   const Workspace &ws, cudaStream_t st, bool outputs = true)
{
    if (p.S > 0) {
        const int rc = launch_all<T, D>(p, q, k, v, beta, M0, z0, out, M_out, z_out, ws, st,
                                        outputs);
        if (rc != INFINI_OK || p.T == 0) return rc;
    }
    return launch_tail<T, D>(p, q, k, v, beta, M0, z0, out, M_out, z_out, st, outputs);
}

// Workspace the chosen path of one forward call needs (p as returned by effective()): the
// fused 64-token paths need far less than the general upper bound workspace_bytes().
template <typename T>
int64_t call_workspace_bytes(const Problem &p)
{
    if (p.S == 0) return 0;
    const int64_t units = p.B * p.Hkv * p.S;
    if (use_small_fused<T>(p)) {
        const int64_t fused = use_pieces(p) ? pieces_workspace_bytes(p) : small_workspace_bytes(p);
        if (p.H == p.Hkv) return fused;
        // grouped heads updated in place take the general (tensor-core) path: room for both
        const int64_t general = tc_workspace_bytes(units, p.d, p.rule == INFINI_UPDATE_DELTA);
        return fused > general ? fused : general;
    }
    return use_tc<T>(p) ? tc_workspace_bytes(units, p.d, p.rule == INFINI_UPDATE_DELTA)
                        : simt_workspace_bytes(units, p.d);
}

// Enqueue the forward (or, with outputs = false, the memory chain alone) on a workspace.
template <typename T>
int dispatch(const Problem &p, const void *q, const void *k, const void *v, const float *beta,
             const float *M0, const float *z0, void *out, float *M_out, float *z_out, void *raw,
             cudaStream_t st, bool outputs = true)
{
    const Workspace ws = carve_workspace(raw, p.B * p.Hkv * p.S, p.d, use_tc<T>(p));
    const T *tq = static_cast<const T *>(q), *tk = static_cast<const T *>(k),
            *tv = static_cast<const T *>(v);
    T *to = static_cast<T *>(out);
    switch (p.d) {
    case 32: return launch_forward<T, 32>(p, tq, tk, tv, beta, M0, z0, to, M_out, z_out, ws, st, outputs);
    case 64: return launch_forward<T, 64>(p, tq, tk, tv, beta, M0, z0, to, M_out, z_out, ws, st, outputs);
    default: return launch_forward<T, 128>(p, tq, tk, tv, beta, M0, z0, to, M_out, z_out, ws, st, outputs);
    }
}

// Test hook (infini_attn_test_fail_allocations): the next n workspace allocations fail as
// if the device were out of memory.
std::atomic<int> g_fail_allocs{0};

bool take_failed_allocation()
{
    int n = g_fail_allocs.load();
    while (n > 0)
        if (g_fail_allocs.compare_exchange_weak(n, n - 1)) return true;
    return false;
}

// The library's own stream-ordered pool on the current device.  Its release threshold keeps
// freed workspace mapped between calls, so a steady stream of same-sized calls does not
// return memory to the driver and map it again every time.
cudaMemPool_t workspace_pool()
{
    constexpr int kMaxDevices = 64;
    static cudaMemPool_t pools[kMaxDevices];
    static std::mutex mu_pool;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> g(mu_pool);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = pool;
    }
    return pools[dev];
}

template <typename T>
int forward(const void *q, const void *k, const void *v, const float *beta, const float *M0,
            const float *z0, void *out, float *M_out, float *z_out, int64_t B, int64_t H,
            int64_t Hkv, int64_t L, int64_t N, int64_t d, int rule, infini_stream_t stream)
{
    Problem p;
    int rc = check_args(q, k, v, beta, M0, z0, out, M_out, z_out, B, H, Hkv, L, N, d, rule,
                        (int64_t)sizeof(T), &p);
    if (rc != INFINI_OK) return rc;
    p = effective<T>(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaGetLastError();   // clear a stale error left by someone else's launch

    const int64_t bytes = call_workspace_bytes<T>(p);
    void *ws = nullptr;
    if (bytes > 0) {
        if (take_failed_allocation()) return INFINI_ERR_OOM;
        cudaMemPool_t pool = workspace_pool();
        if (!pool) return INFINI_ERR_CUDA;
        if (cudaMallocFromPoolAsync(&ws, (size_t)bytes, pool, st) != cudaSuccess) {
            cudaGetLastError();
            return INFINI_ERR_OOM;
        }
    }
    rc = dispatch<T>(p, q, k, v, beta, M0, z0, out, M_out, z_out, ws, st);
    if (ws && cudaFreeAsync(ws, st) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_CUDA;
    return rc;
}

// ---- allocation-free variant of the bf16 forward (workspace: g_noalloc_scratch) ----------
constexpr size_t kNoAllocScratchBytes = (size_t)INFINI_NOALLOC_SCRATCH_BYTES;

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void *noalloc_scratch_address()
{
    constexpr int kMaxDevices = 64;
    static std::atomic<void *> addr[kMaxDevices];
    static std::mutex setup_mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void *a = addr[dev].load(std::memory_order_acquire);
    if (a) return a;
    std::lock_guard<std::mutex> g(setup_mu);
    a = addr[dev].load(std::memory_order_acquire);
    if (a) return a;
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || a == nullptr) {
        cudaGetLastError();
        return nullptr;
    }
    addr[dev].store(a, std::memory_order_release);
    return a;
}

int forward_noalloc(const void *q, const void *k, const void *v, const float *beta,
                    const float *M0, const float *z0, void *out, float *M_out, float *z_out,
                    int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N, int64_t d, int rule,
                    infini_stream_t stream)
{
    using T = __nv_bfloat16;
    Problem p;
    int rc = check_args(q, k, v, beta, M0, z0, out, M_out, z_out, B, H, Hkv, L, N, d, rule,
                        (int64_t)sizeof(T), &p);
    if (rc != INFINI_OK) return rc;
    p = effective<T>(p);
    // admitted by what the chosen path needs (the fused 64-token paths need far less than the
    // general bound infini_attn_workspace_bytes reports)
    const size_t bytes = (size_t)call_workspace_bytes<T>(p);
    if (bytes > kNoAllocScratchBytes) return INFINI_ERR_UNSUPPORTED;
    void *ws = noalloc_scratch_address();
    if (!ws) return INFINI_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaGetLastError();
    // Nothing in the array has to hold anything on entry: every snapshot slot a kernel reads
    // was written earlier in the same call (increments / initial state, then the scan or
    // chain), and the fused 64-token paths clear their tickets and flags first.
    return dispatch<T>(p, q, k, v, beta, M0, z0, out, M_out, z_out, ws, st);
}

// ---- the memory chain alone -----------------------------------------------------------------

// The state after the whole sequence, without the outputs: the forward's memory kernels on
// the same workspace, the segment kernels left out.  Arguments as the forward's, less q,
// beta and out (H is taken as Hkv).
template <typename T>
int state_only(const void *k, const void *v, const float *M0, const float *z0, float *M_out,
               float *z_out, int64_t B, int64_t Hkv, int64_t L, int64_t N, int64_t d, int rule,
               infini_stream_t stream)
{
    if (!k || !v || !M_out || !z_out) return INFINI_ERR_INVALID_ARG;
    // the forward's checks with k standing in for q and out (never written: no outputs) and
    // M_out for beta (never read)
    const int64_t es = (int64_t)sizeof(T), kvbytes = B * Hkv * L * d * es;
    if (B > 0 && Hkv > 0 && L > 0 && d > 0 &&
        (ranges_overlap(M_out, B * Hkv * d * d * 4, k, kvbytes) ||
         ranges_overlap(M_out, B * Hkv * d * d * 4, v, kvbytes) ||
         ranges_overlap(z_out, B * Hkv * d * 4, k, kvbytes) ||
         ranges_overlap(z_out, B * Hkv * d * 4, v, kvbytes)))
        return INFINI_ERR_INVALID_ARG;
    Problem p;
    int rc = check_args(k, k, v, M_out, M0, z0, k, M_out, z_out, B, Hkv, Hkv, L, N, d, rule, es,
                        &p, /*out_checked=*/false);
    if (rc != INFINI_OK) return rc;
    p = effective<T>(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaGetLastError();
    const int64_t units = p.B * p.Hkv * p.S;
    const int64_t bytes = p.S == 0 ? 0
                          : use_tc<T>(p) ? tc_workspace_bytes(units, p.d, p.rule == INFINI_UPDATE_DELTA)
                                         : simt_workspace_bytes(units, p.d);
    void *ws = nullptr;
    if (bytes > 0) {
        if (take_failed_allocation()) return INFINI_ERR_OOM;
        cudaMemPool_t pool = workspace_pool();
        if (!pool) return INFINI_ERR_CUDA;
        if (cudaMallocFromPoolAsync(&ws, (size_t)bytes, pool, st) != cudaSuccess) {
            cudaGetLastError();
            return INFINI_ERR_OOM;
        }
    }
    rc = dispatch<T>(p, k, k, v, nullptr, M0, z0, nullptr, M_out, z_out, ws, st, false);
    if (ws && cudaFreeAsync(ws, st) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_CUDA;
    return rc;
}

// ---- token-by-token decode and the fold of a cached segment -------------------------------

int check_cache_state(const void *k_cache, const void *v_cache, const float *M, const float *z,
                      int64_t B, int64_t Hkv, int64_t N, int64_t d, int rule, int64_t esize)
{
    if (!k_cache || !v_cache || !M || !z) return INFINI_ERR_INVALID_ARG;
    if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return INFINI_ERR_INVALID_ARG;
    if (rule != INFINI_UPDATE_LINEAR && rule != INFINI_UPDATE_DELTA) return INFINI_ERR_INVALID_ARG;
    // grids of up to 8 CTAs per chain stay below 2^31 CTAs
    if (B > (1 << 20) || Hkv > (1 << 16) || B * Hkv > ((int64_t)1 << 27) ||
        N > ((int64_t)1 << 30) || B * Hkv * N > ((int64_t)1 << 40))
        return INFINI_ERR_INVALID_ARG;
    const void *ptrs[] = {k_cache, v_cache, M, z};
    for (const void *p : ptrs)
        if (!aligned16(p)) return INFINI_ERR_INVALID_ARG;
    const int64_t cbytes = B * Hkv * N * d * esize, mbytes = B * Hkv * d * d * 4,
                  zbytes = B * Hkv * d * 4;
    if (ranges_overlap(k_cache, cbytes, v_cache, cbytes) || ranges_overlap(k_cache, cbytes, M, mbytes) ||
        ranges_overlap(k_cache, cbytes, z, zbytes) || ranges_overlap(v_cache, cbytes, M, mbytes) ||
        ranges_overlap(v_cache, cbytes, z, zbytes) || ranges_overlap(M, mbytes, z, zbytes))
        return INFINI_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 128) return INFINI_ERR_UNSUPPORTED;
    return INFINI_OK;
}

template <typename T>
int fold_launch(const void *k_cache, const void *v_cache, int64_t n, float *M, float *z,
                int64_t B, int64_t Hkv, int64_t N, int64_t d, int rule, cudaStream_t st)
{
    const T *kc = static_cast<const T *>(k_cache), *vc = static_cast<const T *>(v_cache);
    const int64_t chains = B * Hkv;
    switch (d) {
    case 32: launch_fold_inplace<T, 32>(kc, vc, N, n, M, z, chains, rule, st); break;
    case 64: launch_fold_inplace<T, 64>(kc, vc, N, n, M, z, chains, rule, st); break;
    default: launch_fold_inplace<T, 128>(kc, vc, N, n, M, z, chains, rule, st); break;
    }
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

template <typename T>
int fold(const void *k_cache, const void *v_cache, int64_t n, float *M, float *z, int64_t B,
         int64_t Hkv, int64_t N, int64_t d, int rule, infini_stream_t stream)
{
    int rc = check_cache_state(k_cache, v_cache, M, z, B, Hkv, N, d, rule, (int64_t)sizeof(T));
    if (rc != INFINI_OK) return rc;
    if (n < 0 || n > N) return INFINI_ERR_INVALID_ARG;
    if (n == 0) return INFINI_OK;
    cudaGetLastError();
    return fold_launch<T>(k_cache, v_cache, n, M, z, B, Hkv, N, d, rule,
                          reinterpret_cast<cudaStream_t>(stream));
}

template <typename T>
int decode_step(const void *q, const void *k, const void *v, const float *beta, void *k_cache,
                void *v_cache, int64_t pos, float *M, float *z, void *out, int64_t B, int64_t H,
                int64_t Hkv, int64_t N, int64_t d, int rule, infini_stream_t stream)
{
    int rc = check_cache_state(k_cache, v_cache, M, z, B, Hkv, N, d, rule, (int64_t)sizeof(T));
    if (rc != INFINI_OK && rc != INFINI_ERR_UNSUPPORTED) return rc;
    const int rc_shape = rc;
    if (!q || !k || !v || !beta || !out) return INFINI_ERR_INVALID_ARG;
    if (H <= 0 || H % Hkv != 0 || H > (1 << 16) || B * H > ((int64_t)1 << 31) - 1)
        return INFINI_ERR_INVALID_ARG;
    if (pos < 0 || pos >= N) return INFINI_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, beta, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return INFINI_ERR_INVALID_ARG;
    const int64_t es = (int64_t)sizeof(T), obytes = B * H * d * es, kvbytes = B * Hkv * d * es,
                  cbytes = B * Hkv * N * d * es;
    if (ranges_overlap(out, obytes, q, obytes) || ranges_overlap(out, obytes, k, kvbytes) ||
        ranges_overlap(out, obytes, v, kvbytes) || ranges_overlap(out, obytes, k_cache, cbytes) ||
        ranges_overlap(out, obytes, v_cache, cbytes) ||
        ranges_overlap(out, obytes, M, B * Hkv * d * d * 4) ||
        ranges_overlap(out, obytes, z, B * Hkv * d * 4))
        return INFINI_ERR_INVALID_ARG;
    if (rc_shape != INFINI_OK) return rc_shape;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaGetLastError();
    const T *tq = static_cast<const T *>(q), *tk = static_cast<const T *>(k),
            *tv = static_cast<const T *>(v);
    T *kc = static_cast<T *>(k_cache), *vc = static_cast<T *>(v_cache), *to = static_cast<T *>(out);
    if (H / Hkv <= kDecodeGMax) {
        // one cluster per (batch, kv head) with its whole query group; a tile of keys per
        // CTA, at most 8 CTAs (the portable cluster size)
        const int KT = sizeof(T) == 2 ? DecCfg<T, 128>::KT : DecCfg<float, 128>::KT;
        const int CL = (int)std::min<int64_t>(8, (pos + KT) / KT);
        size_t smem = 0;
        bool ok = false;
        switch (d) {
        case 32: smem = DecCfg<T, 32>::BYTES; ok = opt_in_smem<k_decode_split<T, 32>>(smem); break;
        case 64: smem = DecCfg<T, 64>::BYTES; ok = opt_in_smem<k_decode_split<T, 64>>(smem); break;
        default: smem = DecCfg<T, 128>::BYTES; ok = opt_in_smem<k_decode_split<T, 128>>(smem); break;
        }
        if (!ok) return INFINI_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(B * Hkv * CL));
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = (unsigned)CL;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        const int ip = (int)pos, iN = (int)N, iH = (int)H, iHkv = (int)Hkv;
        cudaError_t e;
        TRACED("decode_attn", st);
        switch (d) {
        case 32: e = cudaLaunchKernelEx(&cfg, k_decode_split<T, 32>, tq, tk, tv, beta, kc, vc, ip, iN, (const float *)M, (const float *)z, to, iH, iHkv); break;
        case 64: e = cudaLaunchKernelEx(&cfg, k_decode_split<T, 64>, tq, tk, tv, beta, kc, vc, ip, iN, (const float *)M, (const float *)z, to, iH, iHkv); break;
        default: e = cudaLaunchKernelEx(&cfg, k_decode_split<T, 128>, tq, tk, tv, beta, kc, vc, ip, iN, (const float *)M, (const float *)z, to, iH, iHkv); break;
        }
        if (e != cudaSuccess) {
            cudaGetLastError();
            return INFINI_ERR_CUDA;
        }
    } else {   // groups of more than 8 query heads: one CTA per (batch, query head)
        TRACED("decode_attn", st);
        const unsigned grid = (unsigned)(B * H);
        switch (d) {
        case 32: k_decode_attn<T, 32><<<grid, 256, 0, st>>>(tq, tk, tv, beta, kc, vc, (int)pos, (int)N, M, z, to, (int)H, (int)Hkv); break;
        case 64: k_decode_attn<T, 64><<<grid, 256, 0, st>>>(tq, tk, tv, beta, kc, vc, (int)pos, (int)N, M, z, to, (int)H, (int)Hkv); break;
        default: k_decode_attn<T, 128><<<grid, 256, 0, st>>>(tq, tk, tv, beta, kc, vc, (int)pos, (int)N, M, z, to, (int)H, (int)Hkv); break;
        }
    }
    if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_CUDA;
    if (pos + 1 < N) return INFINI_OK;
    return fold_launch<T>(kc, vc, N, M, z, B, Hkv, N, d, rule, st);   // the segment is complete
}

// ---- backward pass --------------------------------------------------------------------------

struct BwdPlan {
    int64_t B, H, Hkv, L, N, d, S, T, chains, units, qtiles;
    int rule;
    bool tc;          // bf16 with d in {64, 128}: the memory path runs on the tensor cores
};

// bf16 activations with d in {64, 128}: the backward's memory recomputation and its
// reverse delta recurrence use the forward's tensor-core memory kernels.
template <typename T>
bool bwd_uses_tc(int64_t d) { return sizeof(T) == 2 && (d == 64 || d == 128); }

// Workspace of one backward call (fp32), in the order carve_bwd lays it out.
int64_t bwd_workspace_bytes(const BwdPlan &p)
{
    const int64_t rows = p.B * p.H * p.L, krows = p.B * p.Hkv * p.L, dd = p.d * p.d;
    const int64_t floats = p.units * dd * 3 + p.units * p.d * 4 + rows * 4 + rows * p.d +
                           p.B * p.H * p.S * p.qtiles + krows * p.d * 3 +
                           (p.tc ? p.units * (p.d + dd + dd + dd / 2) : 0);   // dz, B_s, A_s hi + lo, bf16 M
    return floats * 4 + 20 * 256;
}

BwdWs carve_bwd(void *raw, const BwdPlan &p)
{
    float *f = static_cast<float *>(raw);
    auto take = [&](int64_t n) {
        float *r = f;
        f += (n + 63) / 64 * 64;          // 256-byte aligned pieces
        return r;
    };
    const int64_t rows = p.B * p.H * p.L, krows = p.B * p.Hkv * p.L, dd = p.d * p.d;
    BwdWs w;
    float *snapM = take(p.units * dd), *snapZ = take(p.units * p.d);
    w.snapM = snapM;
    w.snapZ = snapZ;
    w.GM = take(p.units * dd);
    w.dMs = take(p.units * dd);
    w.Gz = take(p.units * p.d);
    w.h = take(p.units * p.d);
    w.dzs = take(p.units * p.d);
    w.lse = take(rows);
    w.Drow = take(rows);
    w.wsc = take(rows);
    w.dden = take(rows);
    w.dq = take(rows * p.d);
    w.dbeta_part = take(p.B * p.H * p.S * p.qtiles);
    w.dk = take(krows * p.d);
    w.dv = take(krows * p.d);
    w.dsk = take(krows * p.d);
    return w;
}

// The tensor-core memory path's buffers of the backward (after carve_bwd's).
Workspace carve_bwd_tc(void *raw, const BwdPlan &p)
{
    const int64_t rows = p.B * p.H * p.L, krows = p.B * p.Hkv * p.L, dd = p.d * p.d;
    int64_t used = 0;
    for (int64_t n : {p.units * dd, p.units * p.d, p.units * dd, p.units * dd, p.units * p.d,
                      p.units * p.d, p.units * p.d, rows, rows, rows, rows, rows * p.d,
                      p.B * p.H * p.S * p.qtiles, krows * p.d, krows * p.d, krows * p.d})
        used += (n + 63) / 64 * 64;
    float *f = static_cast<float *>(raw) + used;
    Workspace w;
    w.raw = raw;
    w.dz = f;
    w.Bs = w.dz + (p.units * p.d + 63) / 64 * 64;
    w.Ahi = reinterpret_cast<__nv_bfloat16 *>(w.Bs + p.units * dd);
    w.Alo = w.Ahi + p.units * dd;
    w.snapMb = w.Alo + p.units * dd;                 // bf16 M_{s-1}, for the row statistics
    return w;
}

template <typename T, int D>
int launch_backward(const BwdPlan &p, const T *q, const T *k, const T *v, const float *beta,
                    const float *M0, const float *z0, const T *dout, const float *dM,
                    const float *dz, T *dq, T *dk, T *dv, float *dbeta, float *dM0, float *dz0,
                    void *raw, cudaStream_t st)
{
    BwdWs w = carve_bwd(raw, p);
    float *snapM = const_cast<float *>(w.snapM), *snapZ = const_cast<float *>(w.snapZ);
    const int S = (int)p.S, N = (int)p.N, T_last = (int)p.T, H = (int)p.H, Hkv = (int)p.Hkv;
    const int64_t chains = p.chains, units = p.units;
    const int64_t per = (int64_t)D * D + D;
    // 1. the memory before every segment (fp32); the final memory goes to scratch (GM, Gz:
    //    overwritten below)
    bool tc_mem = false;
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (p.tc) {
            Workspace tw = carve_bwd_tc(raw, p);
            tw.snapZ = snapZ;
            Problem fp;
            fp.B = p.B; fp.H = p.H; fp.Hkv = p.Hkv; fp.L = p.L; fp.N = p.N; fp.d = p.d;
            fp.S = p.S; fp.Lf = p.S * p.N; fp.T = 0; fp.rule = p.rule;
            const int rc = launch_memory_tc<D>(fp, k, v, M0, z0, tw, w.GM, w.Gz, st, snapM);
            if (rc != INFINI_OK) return rc;
            tc_mem = true;
        }
    }
    if (tc_mem) {
    } else if (p.rule == INFINI_UPDATE_LINEAR) {
        {
            TRACED("bwd_state", st);
            k_linear_increments<T, D><<<(unsigned)units, 256, 0, st>>>(k, v, snapM, snapZ, p.L, N, S,
                                                                       T_last);
        }
        TRACED("bwd_state_scan", st);
        k_linear_scan<<<(unsigned)((chains * per + 255) / 256), 256, 0, st>>>(
            snapM, snapZ, nullptr, M0, z0, w.GM, w.Gz, S, D, chains);
    } else {
        {
            TRACED("bwd_state", st);
            k_state_init<<<(unsigned)((chains * per + 255) / 256), 256, 0, st>>>(M0, z0, snapM, snapZ,
                                                                               nullptr, S, D, chains);
        }
        TRACED("bwd_state_chain", st);
        k_delta_chain<T, D, 16><<<(unsigned)(chains * (D / 16)), 256, 0, st>>>(
            k, v, snapM, snapZ, nullptr, w.GM, nullptr, p.L, N, S, T_last);
    }
    // 2. row statistics, the retrieval part of dq, the gate's partial sums: on the tensor
    //    cores for bf16 with 128-row tiles (the memory path left bf16 snapshots); with
    //    64-token segments (and in step 3) a tile is a pair of segments: the kernels see
    //    N = 128 and ceil(S / 2) segments with `pair` set
    const bool pair = p.N == 64;
    const int Nt = pair ? 128 : N, St = pair ? (S + 1) / 2 : S;
    bool tc_rows = false;
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (tc_mem && (p.N % 128 == 0 || pair)) {
            using CR = tc::BwdRowsCfg<D>;
            Workspace tw = carve_bwd_tc(raw, p);
            CUtensorMap mq, mk, mv, mo, mm;
            if (!make_map_bf16_3d(&mq, q, D, p.L, p.B * p.H, 128) ||
                !make_map_bf16_3d(&mk, k, D, p.L, p.B * p.Hkv, 128) ||
                !make_map_bf16_3d(&mv, v, D, p.L, p.B * p.Hkv, 128) ||
                !make_map_bf16_3d(&mo, dout, D, p.L, p.B * p.H, 128) ||
                !make_map_bf16_3d(&mm, tw.snapMb, D, D, chains * S, D))
                return INFINI_ERR_CUDA;
            if (!opt_in_smem<tc::k_bwd_rows_tc<D>>(CR::ALLOC)) return INFINI_ERR_CUDA;
            tc::BwdRowsArgs ra{beta, snapZ, w.lse, w.Drow, w.wsc, w.dden, w.dq, w.dbeta_part,
                               p.L, Nt, St, H, Hkv, (int)p.qtiles, pair ? 1 : 0, S};
            TRACED("bwd_rows", st);
            tc::k_bwd_rows_tc<D><<<(unsigned)(p.B * p.H * St * (Nt / 128)), 192, CR::ALLOC, st>>>(
                mq, mk, mv, mo, mm, ra);
            tc_rows = true;
        }
    }
    if (!tc_rows) {
        const size_t smem = BwdRowsSmem<D>::bytes;
        if (!opt_in_smem<k_bwd_rows<T, D>>(smem)) return INFINI_ERR_CUDA;
        TRACED("bwd_rows", st);
        k_bwd_rows<T, D><<<(unsigned)(p.B * p.H * S * p.qtiles), 256, smem, st>>>(
            q, k, v, beta, dout, w, p.L, N, S, H, Hkv);
    }
    // 3. dq;  4. local dk, dv: on the tensor cores for bf16 with 128-row tiles
    bool tc_attn = false;
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (p.N % 128 == 0 || pair) {
            using CB = tc::BwdTcCfg<D>;
            CUtensorMap mq, mk, mv, mo;
            if (!make_map_bf16_3d(&mq, q, D, p.L, p.B * p.H, 128) ||
                !make_map_bf16_3d(&mk, k, D, p.L, p.B * p.Hkv, 128) ||
                !make_map_bf16_3d(&mv, v, D, p.L, p.B * p.Hkv, 128) ||
                !make_map_bf16_3d(&mo, dout, D, p.L, p.B * p.H, 128))
                return INFINI_ERR_CUDA;
            if (!opt_in_smem<tc::k_bwd_dq_tc<D>>(CB::ALLOC_DQ) || !opt_in_smem<tc::k_bwd_dkdv_tc<D>>(CB::ALLOC_KV))
                return INFINI_ERR_CUDA;
            tc::BwdTcArgs ta{beta, w.lse, w.Drow, w.dq, reinterpret_cast<__nv_bfloat16 *>(dq), w.dk, w.dv,
                             p.L, Nt, St, H, Hkv, pair ? 1 : 0};
            const int64_t tiles = Nt / 128;
            {
                TRACED("bwd_dq", st);
                tc::k_bwd_dq_tc<D><<<(unsigned)(p.B * p.H * St * tiles), CB::THREADS, CB::ALLOC_DQ, st>>>(
                    mq, mk, mv, mo, ta);
            }
            TRACED("bwd_dkdv", st);
            tc::k_bwd_dkdv_tc<D><<<(unsigned)(chains * St * tiles), CB::THREADS, CB::ALLOC_KV, st>>>(
                mq, mk, mv, mo, ta);
            tc_attn = true;
        }
    }
    if (!tc_attn) {
        const size_t smem = BwdDqSmem<D>::bytes;
        if (!opt_in_smem<k_bwd_dq<T, D>>(smem) || !opt_in_smem<k_bwd_dkdv<T, D>>(smem))
            return INFINI_ERR_CUDA;
        {
            TRACED("bwd_dq", st);
            k_bwd_dq<T, D><<<(unsigned)(p.B * p.H * S * p.qtiles), 256, smem, st>>>(
                q, k, v, beta, dout, w, dq, p.L, N, S, H, Hkv);
        }
        TRACED("bwd_dkdv", st);
        k_bwd_dkdv<T, D><<<(unsigned)(chains * S * p.qtiles), 256, smem, st>>>(
            q, k, v, beta, dout, w, p.L, N, S, H, Hkv);
    }
    // 5. G^M_s, G^z_s (on the tensor cores with the tensor-core row statistics; a 64-token
    //    segment is the first half of the 128-row tile these kernels load, its other rows
    //    count as rows past the segment's end and add nothing);
    // 6. the reverse memory recurrence
    bool tc_gm = false;
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (tc_rows && (p.N % 128 == 0 || pair)) {
            using CG = tc::BwdGmCfg<D>;
            CUtensorMap mq, mo;
            if (!make_map_bf16_3d(&mq, q, D, p.L, p.B * p.H, 128) ||
                !make_map_bf16_3d(&mo, dout, D, p.L, p.B * p.H, 128))
                return INFINI_ERR_CUDA;
            if (!opt_in_smem<tc::k_bwd_gm_tc<D>>(CG::ALLOC)) return INFINI_ERR_CUDA;
            tc::BwdGmArgs ga{w.wsc, w.dden, w.GM, w.Gz, p.L, N, S, H, Hkv};
            TRACED("bwd_gm", st);
            tc::k_bwd_gm_tc<D><<<(unsigned)units, 192, CG::ALLOC, st>>>(mq, mo, ga);
            tc_gm = true;
        }
    }
    if (!tc_gm) {
        TRACED("bwd_gm", st);
        k_bwd_gm<T, D><<<(unsigned)units, 256, 0, st>>>(q, dout, w, p.L, N, S, H, Hkv);
    }
    if (p.rule == INFINI_UPDATE_LINEAR) {
        TRACED("bwd_mem_rev", st);
        k_bwd_mlin<<<(unsigned)((chains * D * D + 255) / 256), 256, 0, st>>>(dM, w, dM0, S, D, chains);
    } else if (tc_mem) {
        // dM_{s-1} = dM_s + G^M_s - A_s dM_s: the forward recurrence run backwards, with the
        // forward's A_s; its snapshots are dM_s, its final state dM0 (scratch: B_s, no longer
        // needed, when the caller does not want it)
        if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
            const Workspace tw = carve_bwd_tc(raw, p);
            using MC = tc::MChainCfg<D>;
            CUtensorMap mah, mal;
            if (!make_map_bf16_3d(&mah, tw.Ahi, D, D, units, D) ||
                !make_map_bf16_3d(&mal, tw.Alo, D, D, units, D))
                return INFINI_ERR_CUDA;
            if (!opt_in_smem<tc::k_mem_chain<D>>(MC::ALLOC)) return INFINI_ERR_CUDA;
            tc::MChainArgs ca{dM, w.GM, nullptr, w.dMs, dM0 ? dM0 : tw.Bs, S, 1};
            TRACED("bwd_mem_rev", st);
            tc::k_mem_chain<D><<<(unsigned)(chains * (D / MC::CB)), MC::THREADS, MC::ALLOC, st>>>(mah, mal, ca);
        }
    } else {
        TRACED("bwd_mem_rev", st);
        k_bwd_mdelta<T, D, 16><<<(unsigned)(chains * (D / 16)), 256, 0, st>>>(k, dM, w, dM0, p.L, N, S);
    }
    // 7. the update's gradients (the same half-tile reading at N = 64);  8. the reverse z
    //    recurrence
    bool tc_upd = false;
    if constexpr (sizeof(T) == 2 && (D == 64 || D == 128)) {
        if (tc_mem && (p.N % 128 == 0 || pair)) {
            using CU = tc::BwdUpdCfg<D>;
            CUtensorMap mk, mv;
            if (!make_map_bf16_3d(&mk, k, D, p.L, p.B * p.Hkv, 128) ||
                !make_map_bf16_3d(&mv, v, D, p.L, p.B * p.Hkv, 128))
                return INFINI_ERR_CUDA;
            tc::BwdUpdArgs ua{w.dMs, snapM, snapZ, w.dv, w.dsk, w.h, p.L, N, S};
            if (p.rule == INFINI_UPDATE_LINEAR) {
                if (!opt_in_smem<tc::k_bwd_update_tc<D, false>>(CU::ALLOC)) return INFINI_ERR_CUDA;
                TRACED("bwd_update", st);
                tc::k_bwd_update_tc<D, false><<<(unsigned)units, 192, CU::ALLOC, st>>>(mk, mv, ua);
            } else {
                if (!opt_in_smem<tc::k_bwd_update_tc<D, true>>(CU::ALLOC)) return INFINI_ERR_CUDA;
                TRACED("bwd_update", st);
                tc::k_bwd_update_tc<D, true><<<(unsigned)units, 192, CU::ALLOC, st>>>(mk, mv, ua);
            }
            tc_upd = true;
        }
    }
    if (!tc_upd) {
        const size_t smem = BwdUpdSmem<D>::bytes;
        if (p.rule == INFINI_UPDATE_LINEAR) {
            if (!opt_in_smem<k_bwd_update<T, D, false>>(smem)) return INFINI_ERR_CUDA;
            TRACED("bwd_update", st);
            k_bwd_update<T, D, false><<<(unsigned)units, 256, smem, st>>>(k, v, w, p.L, N, S);
        } else {
            if (!opt_in_smem<k_bwd_update<T, D, true>>(smem)) return INFINI_ERR_CUDA;
            TRACED("bwd_update", st);
            k_bwd_update<T, D, true><<<(unsigned)units, 256, smem, st>>>(k, v, w, p.L, N, S);
        }
    }
    {
        TRACED("bwd_z_rev", st);
        k_bwd_zrev<<<(unsigned)(chains * ((D + 31) / 32)), 32 * ZREV_CHUNKS, 0, st>>>(dz, w, dz0, S, D,
                                                                                     chains);
    }
    // 9. dk, dv in the activation dtype;  10. dbeta
    {
        const int64_t n = p.B * p.Hkv * p.L * D;
        TRACED("bwd_final", st);
        k_bwd_final<T, D><<<(unsigned)((n / 4 + 255) / 256), 256, 0, st>>>(k, w, dk, dv, p.L, N, S, n);
    }
    if (dbeta) {
        TRACED("bwd_beta", st);
        k_bwd_beta<<<(unsigned)((p.H + 255) / 256), 256, 0, st>>>(w.dbeta_part, dbeta, (int)p.B, H, S,
                                                               (int)p.qtiles);
    }
    return cudaGetLastError() == cudaSuccess ? INFINI_OK : INFINI_ERR_CUDA;
}

template <typename T>
int backward(const void *q, const void *k, const void *v, const float *beta, const float *M0,
             const float *z0, const void *dout, const float *dM, const float *dz, void *dq,
             void *dk, void *dv, float *dbeta, float *dM0, float *dz0, int64_t B, int64_t H,
             int64_t Hkv, int64_t L, int64_t N, int64_t d, int rule, infini_stream_t stream)
{
    if (!q || !k || !v || !beta || !dout || !dq || !dk || !dv) return INFINI_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || Hkv <= 0 || L <= 0 || N <= 0 || d <= 0 || H % Hkv != 0)
        return INFINI_ERR_INVALID_ARG;
    if (rule != INFINI_UPDATE_LINEAR && rule != INFINI_UPDATE_DELTA) return INFINI_ERR_INVALID_ARG;
    if (B > (1 << 20) || H > (1 << 16) || L > ((int64_t)1 << 34) || B * H * L > ((int64_t)1 << 40) ||
        B * H * ((L + 63) / 64) > ((int64_t)1 << 30))
        return INFINI_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, beta, M0, z0, dout, dM, dz, dq, dk, dv, dbeta, dM0, dz0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return INFINI_ERR_INVALID_ARG;
    const int64_t es = (int64_t)sizeof(T), qb = B * H * L * d * es, kb = B * Hkv * L * d * es;
    const int64_t mb = B * Hkv * d * d * 4, zb = B * Hkv * d * 4;
    // outputs overlap no input and no other output
    const void *ins[] = {q, k, v, beta, M0, z0, dout, dM, dz};
    const int64_t insz[] = {qb, kb, kb, H * 4, mb, zb, qb, mb, zb};
    const void *outs[] = {dq, dk, dv, dbeta, dM0, dz0};
    const int64_t outsz[] = {qb, kb, kb, H * 4, mb, zb};
    for (int i = 0; i < 6; ++i) {
        for (int j = 0; j < 9; ++j)
            if (ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return INFINI_ERR_INVALID_ARG;
        for (int j = 0; j < i; ++j)
            if (ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return INFINI_ERR_INVALID_ARG;
    }
    if (d != 32 && d != 64 && d != 128) return INFINI_ERR_UNSUPPORTED;
    if (N % 64 != 0) return INFINI_ERR_UNSUPPORTED;
    BwdPlan p;
    p.B = B; p.H = H; p.Hkv = Hkv; p.L = L; p.N = N; p.d = d;
    p.S = (L + N - 1) / N;
    p.T = L - (p.S - 1) * N;
    p.chains = B * Hkv;
    p.units = p.chains * p.S;
    p.qtiles = N / 64;
    p.rule = rule;
    p.tc = bwd_uses_tc<T>(d);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaGetLastError();
    if (take_failed_allocation()) return INFINI_ERR_OOM;
    cudaMemPool_t pool = workspace_pool();
    if (!pool) return INFINI_ERR_CUDA;
    void *ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, (size_t)bwd_workspace_bytes(p), pool, st) != cudaSuccess) {
        cudaGetLastError();
        return INFINI_ERR_OOM;
    }
    const T *tq = static_cast<const T *>(q), *tk = static_cast<const T *>(k),
            *tv = static_cast<const T *>(v), *tdo = static_cast<const T *>(dout);
    T *gq = static_cast<T *>(dq), *gk = static_cast<T *>(dk), *gv = static_cast<T *>(dv);
    int rc;
    switch (d) {
    case 32: rc = launch_backward<T, 32>(p, tq, tk, tv, beta, M0, z0, tdo, dM, dz, gq, gk, gv, dbeta, dM0, dz0, ws, st); break;
    case 64: rc = launch_backward<T, 64>(p, tq, tk, tv, beta, M0, z0, tdo, dM, dz, gq, gk, gv, dbeta, dM0, dz0, ws, st); break;
    default: rc = launch_backward<T, 128>(p, tq, tk, tv, beta, M0, z0, tdo, dM, dz, gq, gk, gv, dbeta, dM0, dz0, ws, st); break;
    }
    if (cudaFreeAsync(ws, st) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_CUDA;
    return rc;
}

}  // namespace
}  // namespace infini

extern "C" {

int infini_attn_fwd_noalloc(const void *q, const void *k, const void *v, const float *beta,
                            const float *M0, const float *z0, void *out, float *M_out,
                            float *z_out, int64_t B, int64_t H, int64_t Hkv, int64_t L,
                            int64_t N, int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::forward_noalloc(q, k, v, beta, M0, z0, out, M_out, z_out, B, H, Hkv, L, N, d,
                                   update_rule, stream);
}

int infini_attn_fwd(const void *q, const void *k, const void *v, const float *beta,
                    const float *M0, const float *z0, void *out, float *M_out, float *z_out,
                    int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N, int64_t d,
                    int update_rule, infini_stream_t stream)
{
    return infini::forward<__nv_bfloat16>(q, k, v, beta, M0, z0, out, M_out, z_out, B, H, Hkv,
                                          L, N, d, update_rule, stream);
}

int infini_attn_bwd(const void *q, const void *k, const void *v, const float *beta,
                    const float *M0, const float *z0, const void *dout, const float *dM,
                    const float *dz, void *dq, void *dk, void *dv, float *dbeta, float *dM0,
                    float *dz0, int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N,
                    int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::backward<__nv_bfloat16>(q, k, v, beta, M0, z0, dout, dM, dz, dq, dk, dv, dbeta,
                                           dM0, dz0, B, H, Hkv, L, N, d, update_rule, stream);
}

int infini_attn_bwd_f32(const void *q, const void *k, const void *v, const float *beta,
                        const float *M0, const float *z0, const void *dout, const float *dM,
                        const float *dz, void *dq, void *dk, void *dv, float *dbeta, float *dM0,
                        float *dz0, int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N,
                        int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::backward<float>(q, k, v, beta, M0, z0, dout, dM, dz, dq, dk, dv, dbeta, dM0,
                                   dz0, B, H, Hkv, L, N, d, update_rule, stream);
}

int infini_attn_fwd_f32(const void *q, const void *k, const void *v, const float *beta,
                        const float *M0, const float *z0, void *out, float *M_out,
                        float *z_out, int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N,
                        int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::forward<float>(q, k, v, beta, M0, z0, out, M_out, z_out, B, H, Hkv, L, N, d,
                                  update_rule, stream);
}

int infini_attn_state(const void *k, const void *v, const float *M0, const float *z0,
                      float *M_out, float *z_out, int64_t B, int64_t Hkv, int64_t L, int64_t N,
                      int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::state_only<__nv_bfloat16>(k, v, M0, z0, M_out, z_out, B, Hkv, L, N, d,
                                             update_rule, stream);
}

int infini_attn_state_f32(const void *k, const void *v, const float *M0, const float *z0,
                          float *M_out, float *z_out, int64_t B, int64_t Hkv, int64_t L,
                          int64_t N, int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::state_only<float>(k, v, M0, z0, M_out, z_out, B, Hkv, L, N, d, update_rule,
                                     stream);
}

int infini_attn_decode_step(const void *q, const void *k, const void *v, const float *beta,
                            void *k_cache, void *v_cache, int64_t pos, float *M, float *z,
                            void *out, int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                            int update_rule, infini_stream_t stream)
{
    return infini::decode_step<__nv_bfloat16>(q, k, v, beta, k_cache, v_cache, pos, M, z, out, B,
                                              H, Hkv, N, d, update_rule, stream);
}

int infini_attn_decode_step_f32(const void *q, const void *k, const void *v, const float *beta,
                                void *k_cache, void *v_cache, int64_t pos, float *M, float *z,
                                void *out, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                                int64_t d, int update_rule, infini_stream_t stream)
{
    return infini::decode_step<float>(q, k, v, beta, k_cache, v_cache, pos, M, z, out, B, H, Hkv,
                                      N, d, update_rule, stream);
}

int infini_attn_fold(const void *k_cache, const void *v_cache, int64_t n, float *M, float *z,
                     int64_t B, int64_t Hkv, int64_t N, int64_t d, int update_rule,
                     infini_stream_t stream)
{
    return infini::fold<__nv_bfloat16>(k_cache, v_cache, n, M, z, B, Hkv, N, d, update_rule,
                                       stream);
}

int infini_attn_fold_f32(const void *k_cache, const void *v_cache, int64_t n, float *M, float *z,
                         int64_t B, int64_t Hkv, int64_t N, int64_t d, int update_rule,
                         infini_stream_t stream)
{
    return infini::fold<float>(k_cache, v_cache, n, M, z, B, Hkv, N, d, update_rule, stream);
}

int64_t infini_attn_workspace_bytes(int64_t B, int64_t Hkv, int64_t L, int64_t N, int64_t d)
{
    if (B <= 0 || Hkv <= 0 || L <= 0 || N <= 0 || d <= 0) return 0;
    return infini::workspace_bytes(B, Hkv, L, N, d);
}

const char *infini_attn_status_string(int status)
{
    switch (status) {
    case INFINI_OK: return "ok";
    case INFINI_ERR_INVALID_ARG: return "invalid argument";
    case INFINI_ERR_UNSUPPORTED: return "unsupported shape (d must be 32, 64 or 128; N a multiple of 64)";
    case INFINI_ERR_CUDA: return "CUDA error";
    case INFINI_ERR_OOM: return "workspace allocation failed";
    case INFINI_ERR_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
    }
}

int infini_attn_version(void) { return 100; }

int infini_attn_device_status(infini_stream_t stream)
{
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return INFINI_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, infini::tc::g_wait_status, sizeof(int)) != cudaSuccess)
        return INFINI_ERR_CUDA;
    if (v == 0) return INFINI_OK;
    const int zero = 0;
    cudaMemcpyToSymbol(infini::tc::g_wait_status, &zero, sizeof(int));
    return INFINI_ERR_TIMEOUT;
}

int infini_attn_test_fail_allocations(int n)
{
    if (n < 0) return INFINI_ERR_INVALID_ARG;
    infini::g_fail_allocs.store(n);
    return INFINI_OK;
}

int infini_attn_test_wait_limit(int64_t cycles)
{
    const long long v = cycles > 0 ? (long long)cycles : infini::tc::kSpinLimitCycles;
    return cudaMemcpyToSymbol(infini::tc::g_spin_limit, &v, sizeof(v)) == cudaSuccess
        ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_test_withhold_publish(int on)
{
    const int v = on ? 1 : 0;
    return cudaMemcpyToSymbol(infini::tc::g_test_withhold, &v, sizeof(v)) == cudaSuccess
        ? INFINI_OK : INFINI_ERR_CUDA;
}

int infini_attn_trace_enable(int on)
{
    using namespace infini::trace;
    std::lock_guard<std::mutex> g(mu);
    if (on) {   // a new trace: drop pending records and the accumulated table
        for (const Rec &r : recs) {
            cudaEventSynchronize(r.b);
            give_event(r.a);
            give_event(r.b);
        }
        recs.clear();
        names.clear();
        counts.clear();
        ms.clear();
        failed = false;
    }
    return enabled.exchange(on ? 1 : 0);
}

int64_t infini_attn_trace_report(char *buf, int64_t len)
{
    using namespace infini::trace;
    std::lock_guard<std::mutex> g(mu);
    // fold pending records into the per-kernel table (first-seen order)
    for (const Rec &r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            failed = true;
        give_event(r.a);
        give_event(r.b);
        size_t i = 0;
        while (i < names.size() && names[i] != r.name) ++i;
        if (i == names.size()) {
            names.emplace_back(r.name);
            counts.push_back(0);
            ms.push_back(0.0);
        }
        counts[i] += 1;
        ms[i] += t;
    }
    recs.clear();
    std::string js = "{";
    for (size_t i = 0; i < names.size(); ++i) {
        char item[160];
        snprintf(item, sizeof(item), "%s\"%s\": {\"launches\": %lld, \"ms\": %.6f}", i ? ", " : "",
                 names[i].c_str(), (long long)counts[i], ms[i]);
        js += item;
    }
    if (failed) js += names.empty() ? "\"error\": true" : ", \"error\": true";
    js += "}";
    if (buf && len > 0) {
        const size_t n = js.size() < (size_t)(len - 1) ? js.size() : (size_t)(len - 1);
        memcpy(buf, js.data(), n);
        buf[n] = 0;
    }
    return (int64_t)js.size() + 1;
}

}  // extern "C"
