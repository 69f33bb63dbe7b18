// select.cu -- RPCholesky coreset selection on sm_100a.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2
// (randomly pivoted Cholesky; Alg. 1 RPNys).  For each instance, r
// sequential steps:
//   draw s with probability proportional to the residual diagonal d,
//   g = h(K, k_s) - F[:, :i] F[s, :i]^T,   h(x, y) = exp(beta (<x,y> - M_K)),
//   F[:, i] = g / sqrt(g_s),   d <- max(d - F[:, i]^2, 0),   d_s = 0,
// stopping early when the total mass or the pivot residual g_s vanishes.
//
// Mapping: one thread-block cluster of G CTAs per instance.  CTA c owns the
// key rows [c R, c R + R).  It keeps the residual diagonal of its rows in
// shared memory (double-buffered across steps) together with fp64 chunk sums
// of it; the pivot search reads the other CTAs' chunk sums and the chosen
// chunk through distributed shared memory, so the cluster needs one
// hardware cluster barrier per step.  Every CTA runs the search on the same
// data with the same arithmetic, so all CTAs agree on s without a second
// barrier.  The column pass streams the CTA's slice of F[:, :i] (float4,
// L2-only loads: the slice is touched once per step) and of K, spread over
// JG thread groups that split the factor columns and the head dimension.
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "internal.h"
#include "philox.cuh"

namespace cg = cooperative_groups;

namespace wildcat {

namespace {

constexpr int kFsByWarp0 = 512;  // factor rows up to this length are gathered by warp 0 alone
constexpr int kMaxPL = 16;  // R <= 16384 rows per CTA -> at most 16 values per lane
constexpr size_t kSmemCap = 227 * 1024;
constexpr int kGsMaxCtas = 160;  // global-sync CTAs per instance (the search gives a lane ceil(G / 32))

struct SelectArgs {
    const void* K;
    int64_t BH, n;
    float beta;
    int r;
    uint64_t seed;
    int64_t inst0;           // global index of instance 0 (Philox counter word 1 = inst0 + b)
    const float* kbar;       // per-instance key mean subtracted from every key (or nullptr)
    int kbar_div;            // instance b uses kbar row b / kbar_div (bins of one instance share it)
    float eps;
    const int32_t* S_fixed;  // nullptr: draw pivots
    int32_t* S;              // may be nullptr in fixed mode
    float* F;
    int32_t* rank;
    void* K_S;  // may be nullptr
    int G;      // CTAs per instance (cluster size)
    int R;      // rows per CTA, multiple of 4
    int JG;     // thread groups splitting factor columns / head dim
    int PL;     // residual values per lane in one search chunk (multiple of 4)
    // global-sync mode (the CTAs of an instance are not a cluster): exchange buffers
    double* gs_inbox;  // [BH][2][G][33] chunk sums + total per CTA
    float* gs_resid;   // [BH][2][G][Rpad] residual diagonal copies
    unsigned* gs_bar;  // [BH] barrier counters, zero at launch
    float* gs_mk;      // [BH][G] per-CTA max |k|^2
    int gs;            // 1: the launch is the global-sync one
    unsigned long long gs_force_ns;  // test hook: CTA 0 of each instance skips barrier 2; waits end after this
    // phases: the launch runs steps [step0, step_end); an instance still going at
    // step_end saves its residual diagonal and joins the list of the next phase
    int step0, step_end;
    float* ph_resid;       // [BH][n] residual diagonal of paused instances
    float* ph_mk;          // [BH] M_K (written by the first phase)
    const int* act_in;     // resumed launch (global sync): instances to continue, count at act_n_in
    const int* act_n_in;
    int* act_out;          // instances paused at step_end (order of arrival), count at act_n_out
    int* act_n_out;
    int grid_ctas;         // resumed launch: CTAs of the grid (else BH G)
};

// Rows per CTA, thread groups and search-chunk width for G CTAs per instance
// (host plan and the resumed launch's per-phase choice use the same rule).
struct SelectShape {
    int R, JG, PL, Rpad;
    __host__ __device__ SelectShape(int64_t n, int G, int nt, int vec) {
        R = (int)round_up(ceil_div(n, G), 4);
        JG = 1;
        while (JG * 2 <= 8 && (int64_t)(nt / (JG * 2)) * vec >= R) JG *= 2;
        const int64_t pl = round_up(ceil_div(ceil_div(R, 32), 32), 4);
        PL = (int)(pl > 4 ? pl : 4);
        Rpad = (int)round_up(R, 32 * PL);
    }
};

struct SmemLayout {
    size_t ring, kres, inbox, csl, dbuf, dotb, ks, fs, red, misc, total;
    __host__ __device__ SmemLayout(int Rpad, int r, int D, int JG, int NT, int VEC, int G, int depth,
                                   size_t kres_bytes, bool gs = false) {
        size_t o = 0;
        ring = o;  o += (size_t)depth * NT * 16;               // per-thread cp.async ring, [slot][thread] x 16 B
        kres = o;  o += round_up(kres_bytes, 16);              // the CTA's key rows, when resident
        inbox = o; o += gs ? 0 : 2 * (size_t)G * 33 * sizeof(double);  // [parity][source CTA][32 chunk sums + total]
        csl = o;   o += 32 * sizeof(double);                   // own chunk sums
        dbuf = o;  o += 2 * (size_t)Rpad * sizeof(float);      // residual diagonal, double-buffered
        dotb = o;  o += (size_t)Rpad * sizeof(float);          // <k_l, k_s> of the step
        ks = o;    o += (size_t)D * sizeof(float);
        fs = o;    o += (size_t)round_up(r, 4) * sizeof(float);
        o = round_up(o, 16);
        red = o;   o += (size_t)(JG > 1 ? JG - 1 : 0) * (NT / JG) * VEC * sizeof(float);
        misc = o;  o += 16 * sizeof(float);
        total = round_up(o, 16);
    }
};

// Inclusive fp64 warp scan (Hillis-Steele); identical on every CTA.
__device__ __forceinline__ double warp_scan_incl(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Sum of one search chunk (PL values per lane, lane-sequential then scan).
__device__ __forceinline__ double chunk_total(const float* chunk, int PL, int lane) {
    double s = 0.0;
    for (int k = 0; k < PL; ++k) s += (double)chunk[lane * PL + k];
    return __shfl_sync(0xffffffffu, warp_scan_incl(s, lane), 31);
}

// Global-sync mode helpers: acquire load of a barrier counter, the clock for
// the bounded wait, and the status word a timed-out wait records.
constexpr unsigned long long kGsWaitNs = 2000000000ull;
__device__ int g_select_gs_status = 0;
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long gs_clock() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One lane's share of a key-row dot product: 16 bytes of the row (EPL
// elements) against x.  Without recentring the pairs go through the packed
// fp32x2 FMA (two partial sums); with it every element is shifted first.
__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) {
    unsigned long long A = *reinterpret_cast<unsigned long long*>(&a);
    unsigned long long B = *reinterpret_cast<unsigned long long*>(&b);
    unsigned long long C = *reinterpret_cast<unsigned long long*>(&acc);
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(C) : "l"(A), "l"(B));
    acc = *reinterpret_cast<float2*>(&C);
}

template <typename T, int EPL, bool KB>
__device__ __forceinline__ float lane_dot(const float4& raw, const float (&x)[EPL], const float (&kbr)[EPL]) {
    if constexpr (!KB) {
        float2 acc = make_float2(0.f, 0.f);
        if constexpr (sizeof(T) == 2) {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 v = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
                ffma2(acc, v, make_float2(x[2 * k], x[2 * k + 1]));
            }
        } else {
            ffma2(acc, make_float2(raw.x, raw.y), make_float2(x[0], x[1]));
            ffma2(acc, make_float2(raw.z, raw.w), make_float2(x[2], x[3]));
        }
        return acc.x + acc.y;
    } else {
        float v[EPL];
        if constexpr (sizeof(T) == 2) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(h[k]);
                v[2 * k] = f.x;
                v[2 * k + 1] = f.y;
            }
        } else {
            v[0] = raw.x; v[1] = raw.y; v[2] = raw.z; v[3] = raw.w;
        }
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) part = fmaf(v[e] - kbr[e], x[e], part);
        return part;
    }
}

// cp.async helpers (16-byte copies global -> shared, L2 only)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <typename E, int D, int VEC, int DEPTH, int KM, bool GS, int NTH>
__global__ void __launch_bounds__(NTH, 512 / NTH) rpc_select_kernel(const SelectArgs a) {
    // NTH threads per CTA: 512 (one CTA per SM), or 256 with twice the CTAs
    // per instance and two CTAs per SM, whose barriers and searches overlap.
    // KM: 0 keys streamed each step, 1 keys resident in shared memory.
    constexpr bool KRES = KM >= 1;
    // Launched with a cluster dimension of a.G (one cluster per instance), or,
    // with GS, as one cooperative grid whose a.G CTAs per instance exchange
    // chunk sums and residuals through global memory and meet at a counter
    // barrier (all CTAs are co-resident by the cooperative launch).
    using T = typename E::T;
    constexpr int NT = NTH, NW = NT / 32;
    constexpr int EPL = 16 / (int)sizeof(T);  // key elements per 16-byte load
    constexpr int LPR = D / EPL;              // lanes per key row
    constexpr int RPW = 32 / LPR;             // key rows per warp-wide load
    constexpr int UF = 8;                     // factor loads in flight per thread (scalar path)
    cg::cluster_group cluster = cg::this_cluster();
    int G = a.G, R = a.R, JG = a.JG, PL = a.PL;
    int64_t b;
    int crank;
    const bool resume = GS && a.act_in != nullptr;
    if (resume) {
        // a resumed phase: the A instances still going share the grid, each
        // with as many CTAs as fit (a.G is the least the host planned for)
        const int A = *a.act_n_in;
        if (A <= 0) return;
        int g = (int)(gridDim.x / (unsigned)A);
        g = g < kGsMaxCtas ? g : kGsMaxCtas;
        // at least 256 rows per CTA (late steps stream 4 i bytes per row)
        const int64_t by_rows = a.n / 256;
        g = (int64_t)g < by_rows ? g : (int)(by_rows > 1 ? by_rows : 1);
        G = g > a.G ? g : a.G;
        const SelectShape sh(a.n, G, NTH, VEC);
        R = sh.R;
        JG = sh.JG;
        PL = sh.PL;
        const int slot = (int)(blockIdx.x / (unsigned)G);
        if (slot >= A) return;  // whole groups only
        b = a.act_in[slot];
        crank = (int)(blockIdx.x % (unsigned)G);
    } else {
        crank = GS ? (int)(blockIdx.x % a.G) : (int)cluster.block_rank();
        b = blockIdx.x / a.G;
        if (b >= a.BH) return;  // whole clusters only: G divides gridDim.x
    }

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = a.r, TPG = NT / JG;
    const int64_t n = a.n;
    const int64_t row0 = (int64_t)crank * R;
    const int64_t row_end = (row0 + R < n) ? row0 + R : n;
    const int nrows = row_end > row0 ? (int)(row_end - row0) : 0;
    const int CH = 32 * PL;
    const int nch = (int)ceil_div(R, CH);
    const int Rpad = nch * CH;  // residual buffers cover whole search chunks

    extern __shared__ __align__(16) unsigned char smem[];
    const SmemLayout L(Rpad, r, D, JG, NT, VEC, G, DEPTH, KRES ? (size_t)R * D * sizeof(T) : 0, GS);
    // Each thread streams through its own DEPTH slots of 16 bytes
    // (slot q of thread t at ring4[q * NT + t]); it only ever reads slots it
    // filled itself, so the pipeline needs no barrier.  A slot is refilled
    // two iterations after it was read, keeping DEPTH - 2 copies in flight.
    float4* ring4 = reinterpret_cast<float4*>(smem + L.ring) + tid;
    constexpr int INFL = DEPTH - 2;
    double* inbox = reinterpret_cast<double*>(smem + L.inbox);
    double* csl = reinterpret_cast<double*>(smem + L.csl);
    float* dbuf = reinterpret_cast<float*>(smem + L.dbuf);
    float* dotb = reinterpret_cast<float*>(smem + L.dotb);
    float* fs = reinterpret_cast<float*>(smem + L.fs);
    T* ksm = reinterpret_cast<T*>(smem + L.ks);  // the pivot's key row (D elements)
    float* red = reinterpret_cast<float*>(smem + L.red);
    float* misc = reinterpret_cast<float*>(smem + L.misc);
    int* imisc = reinterpret_cast<int*>(misc);
    // misc[0] local max |k|^2, misc[1] M_K, misc[2] g_s, imisc[3] s, imisc[4] stop, imisc[5] abort (GS)

    // Global-sync mode: the instance's barrier is a counter in global memory;
    // barrier k completes when all G CTAs have added one for it.  The wait is
    // bounded (2 s): on expiry the CTA records WILDCAT_ERR_TIMEOUT and stops
    // (its peers then run out at their next barrier).  Peer data is read with
    // L2-only loads after the barrier.
    int gs_k = 0;
    auto gsync = [&]() -> bool {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const bool skip = a.gs_force_ns && gs_k == 2 && crank == 0;  // test hook: never arrive
            if (!skip) atomicAdd(a.gs_bar + b, 1u);
            const unsigned target = (unsigned)G * (unsigned)(gs_k + 1);
            const unsigned long long limit = a.gs_force_ns ? a.gs_force_ns : kGsWaitNs;
            const unsigned long long t0 = gs_clock();
            while (ld_acquire_u32(a.gs_bar + b) < target) {
                if (gs_clock() - t0 > limit) {
                    imisc[5] = 1;
                    atomicExch(&g_select_gs_status, 5);
                    break;
                }
            }
            __threadfence();
        }
        ++gs_k;
        __syncthreads();
        return imisc[5] == 0;
    };
    if (GS && tid == 0) imisc[5] = 0;
    auto ginbox = [&](int par, int c) -> double* { return a.gs_inbox + (((size_t)b * 2 + par) * G + c) * 33; };
    auto gres = [&](int par) -> float* { return a.gs_resid + (((size_t)b * 2 + par) * G + crank) * (size_t)Rpad; };

    const T* Kb = reinterpret_cast<const T*>(a.K) + b * n * D;
    float* Fb = a.F + b * (int64_t)r * n;
    const int kl_row = lane / LPR, kl_part = lane % LPR;

    // Warp-cooperative pass over the CTA's key rows: out[row] = <k_row, x>
    // (x = ks) or |k_row|^2 (x = nullptr).  LPR lanes share one row, each
    // copying 16 contiguous bytes, so a warp reads RPW whole rows per item;
    // items stream through the thread's cp.async ring.
    // 16-byte piece pc of resident key row `row` (row-major)
    auto kres_off = [&](int row, int pc) -> size_t { return ((size_t)row * D + pc * EPL) * sizeof(T); };
    // Recentring: every key enters as k - kbar (kbar = 0 without recentring,
    // which leaves the arithmetic bit-identical).
    float kbr[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e)
        kbr[e] = a.kbar ? a.kbar[(b / a.kbar_div) * D + kl_part * EPL + e] : 0.f;
    const bool has_kbar = a.kbar != nullptr;
    // The first INFL items of the streamed key pass.
    const int kfirst = warp * RPW + kl_row;  // row of item 0 for this lane
    const int kitems = nrows > warp * RPW ? (int)ceil_div(nrows - warp * RPW, NW * RPW) : 0;  // warp-uniform
    const T* ksrc0 = Kb + (row0 + kfirst) * D + kl_part * EPL;
    const int64_t kstep = (int64_t)NW * RPW * D;
    auto key_prime = [&]() {
#pragma unroll
        for (int q = 0; q < INFL; ++q) {
            if (q < kitems && kfirst + q * NW * RPW < nrows) cp_async16(ring4 + q * NT, ksrc0 + q * kstep);
            cp_async_commit();
        }
    };
    // out[row] = <k_row - kbar, x> (or |k_row - kbar|^2 when self)
    auto key_pass = [&](const float (&x)[EPL], bool self, float* out) {
        if constexpr (KRES) {
            // key rows resident in shared memory: no global traffic; four rows per lane in flight
            for (int base = warp * RPW; base < nrows; base += 4 * NW * RPW) {
                float part[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int row = base + u * NW * RPW + kl_row;
                    part[u] = 0.f;
                    if (row < nrows) {
                        const float4 raw = *reinterpret_cast<const float4*>(smem + L.kres + kres_off(row, kl_part));
                        if (self) {
                            float v[EPL];
                            if constexpr (sizeof(T) == 2) {
                                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const float2 f = __bfloat1622float2(h[k]);
                                    v[2 * k] = f.x;
                                    v[2 * k + 1] = f.y;
                                }
                            } else {
                                v[0] = raw.x; v[1] = raw.y; v[2] = raw.z; v[3] = raw.w;
                            }
#pragma unroll
                            for (int e = 0; e < EPL; ++e) v[e] -= kbr[e];
#pragma unroll
                            for (int e = 0; e < EPL; ++e) part[u] = fmaf(v[e], v[e], part[u]);
                        } else {
                            part[u] = has_kbar ? lane_dot<T, EPL, true>(raw, x, kbr) : lane_dot<T, EPL, false>(raw, x, kbr);
                        }
                    }
                }
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1)
#pragma unroll
                    for (int u = 0; u < 4; ++u) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
                if (kl_part == 0) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int row = base + u * NW * RPW + kl_row;
                        if (row < nrows) out[row] = part[u];
                    }
                }
            }
            return;
        }
        key_prime();
        // slot and source advance incrementally (no division or 64-bit multiply per item)
        int slot_rd = 0, slot_wr = INFL;
        const T* src_wr = ksrc0 + INFL * kstep;
        int row_wr = kfirst + INFL * NW * RPW;
        for (int q = 0; q < kitems; ++q) {
            if (q + INFL < kitems && row_wr < nrows) cp_async16(ring4 + slot_wr * NT, src_wr);
            cp_async_commit();
            src_wr += kstep;
            row_wr += NW * RPW;
            slot_wr = slot_wr + 1 == DEPTH ? 0 : slot_wr + 1;
            cp_async_wait<INFL>();
            const int row = kfirst + q * NW * RPW;
            float part = 0.f;
            const float4 raw = ring4[slot_rd * NT];
            slot_rd = slot_rd + 1 == DEPTH ? 0 : slot_rd + 1;
            if (row < nrows) {
                if (self) {
                    float v[EPL];
                    if constexpr (sizeof(T) == 2) {
                        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 f = __bfloat1622float2(h[k]);
                            v[2 * k] = f.x;
                            v[2 * k + 1] = f.y;
                        }
                    } else {
                        v[0] = raw.x; v[1] = raw.y; v[2] = raw.z; v[3] = raw.w;
                    }
#pragma unroll
                    for (int e = 0; e < EPL; ++e) v[e] -= kbr[e];
#pragma unroll
                    for (int e = 0; e < EPL; ++e) part = fmaf(v[e], v[e], part);
                } else {
                    part = has_kbar ? lane_dot<T, EPL, true>(raw, x, kbr) : lane_dot<T, EPL, false>(raw, x, kbr);
                }
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (kl_part == 0 && row < nrows) out[row] = part;
        }
        cp_async_wait<0>();
    };

    // Chunk sums of a freshly written residual buffer (unless the epilogue
    // formed them), pushed with the CTA total into every peer's
    // inbox[par][crank]; the cluster barrier is split so that warp 0 draws
    // the next step's uniform while the cluster arrives.
    double u_next = 0.0;  // warp 0: the uniform of the next step
    auto publish = [&](const float* dnew, int par, bool have_csl, int next_step) {
        if (!have_csl) {
            for (int k = warp; k < nch; k += NW) {
                const double t = chunk_total(dnew + (size_t)k * CH, PL, lane);
                if (lane == 0) csl[k] = t;
            }
            __syncthreads();
        }
        if constexpr (GS) {
            if (warp == 0) {
                const double v = lane < nch ? csl[lane] : 0.0;
                const double tot = __shfl_sync(0xffffffffu, warp_scan_incl(v, lane), 31);
                double* dst = ginbox(par, crank);
                if (lane < nch) dst[lane] = v;
                if (lane == 0) dst[32] = tot;
                u_next = pivot_uniform(a.seed, (uint32_t)next_step, (uint32_t)(a.inst0 + b));
            }
            gsync();
        } else {
            if (warp == 0) {
                const double v = lane < nch ? csl[lane] : 0.0;
                const double tot = __shfl_sync(0xffffffffu, warp_scan_incl(v, lane), 31);
                for (int c = 0; c < G; ++c) {
                    double* dst = cluster.map_shared_rank(inbox + ((size_t)par * G + crank) * 33, c);
                    if (lane < nch) dst[lane] = v;
                    if (lane == 0) dst[32] = tot;
                }
            }
            cluster.barrier_arrive();
            if (warp == 0) u_next = pivot_uniform(a.seed, (uint32_t)next_step, (uint32_t)(a.inst0 + b));
            cluster.barrier_wait();
        }
    };

    // ---------------- prologue: M_K and the initial residual diagonal ----------------
    // (a resumed phase reads both back instead)
    const int step0 = a.step0;
    float MK;
    if (resume) {
        if (tid == 0) misc[1] = a.ph_mk[b];
        const float* src = a.ph_resid + b * n + row0;
        float* d0 = dbuf + (size_t)(step0 & 1) * Rpad;
        for (int row = tid; row < Rpad; row += NT) {
            const float v = row < nrows ? __ldcg(src + row) : 0.f;
            d0[row] = v;
            gres(step0 & 1)[row] = v;
        }
        __syncthreads();
        MK = misc[1];
        publish(d0, step0 & 1, false, step0);
    } else {
    if constexpr (KRES) {
        const int pieces = nrows * LPR;
        for (int c = tid; c < pieces; c += NT) {
            const int row = c / LPR, pc = c % LPR;
            cp_async16(smem + L.kres + kres_off(row, pc), Kb + (row0 + row) * D + pc * EPL);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
    }
    {
        const float none[EPL] = {};
        key_pass(none, true, dotb);  // |k_l - kbar|^2
    }
    __syncthreads();
    float lmax = -INFINITY;
    for (int row = tid; row < nrows; row += NT) lmax = fmaxf(lmax, dotb[row]);
    lmax = warp_max(lmax);
    __shared__ float wmax[NW];
    if (lane == 0) wmax[warp] = lmax;
    __syncthreads();
    if (warp == 0) {
        float v = lane < NW ? wmax[lane] : -INFINITY;
        v = warp_max(v);
        if (lane == 0) misc[0] = v;
    }
    if constexpr (GS) {
        if (tid == 0) a.gs_mk[b * G + crank] = misc[0];
        gsync();
        if (warp == 0) {
            float v = -INFINITY;
            for (int c = lane; c < G; c += 32) v = fmaxf(v, __ldcg(a.gs_mk + b * G + c));
            v = warp_max(v);
            if (lane == 0) misc[1] = v;
        }
    } else {
        cluster.sync();
        if (warp == 0) {
            float v = -INFINITY;
            if (lane < G) v = *cluster.map_shared_rank(&misc[0], lane);
            v = warp_max(v);
            if (lane == 0) misc[1] = v;
        }
    }
    __syncthreads();
    MK = misc[1];
    if (a.ph_mk && crank == 0 && tid == 0) a.ph_mk[b] = MK;
    for (int row = tid; row < Rpad; row += NT) {
        const float v = row < nrows ? expf(a.beta * (dotb[row] - MK)) : 0.f;
        dbuf[row] = v;
        if constexpr (GS) gres(0)[row] = v;
    }
    __syncthreads();
    publish(dbuf, 0, false, 0);
    }
    const float beta = a.beta;
    const bool gs_ok = !(GS && imisc[5]);

    // ---------------- r sequential steps ----------------
    // The epilogue forms the search's chunk sums itself when a chunk is
    // exactly one warp's rows (4 per lane): then group-0 warp w of a row
    // block covers chunk (base + 128 w) / 128 with the search's lane layout.
    const bool fused_csl = (VEC == 4 && PL == 4);
    const int g = tid / TPG, tt = tid % TPG;
    const int step_end = a.step_end;
    int i = step0;
    for (; gs_ok && i < step_end; ++i) {
        // a barrier ran out: the steps before it are complete (uniform: read after the barrier's block sync)
        if (GS && imisc[5]) break;
        const int cur = i & 1, nxt = cur ^ 1;
        float* dcur = dbuf + (size_t)cur * Rpad;
        float* dnxt = dbuf + (size_t)nxt * Rpad;
        const double* ib = inbox + (size_t)cur * G * 33;

        // -- pivot search (warp 0 of every CTA, identical arithmetic) --
        if (warp == 0) {
            int s = -1;
            if (a.S_fixed) {
                const int sf = a.S_fixed[b * r + i];
                s = (sf >= 0 && (int64_t)sf < n) ? sf : -1;
            } else {
                // CTA totals, CPL consecutive CTAs per lane (one unless a global-sync
                // launch has more than 32 CTAs per instance; clusters have at most 16)
                const int CPL = GS ? (G + 31) >> 5 : 1;
                auto cta_total = [&](int c) -> double {
                    return c < G ? (GS ? __ldcg(ginbox(cur, c) + 32) : ib[c * 33 + 32]) : 0.0;
                };
                double tc = cta_total(lane * CPL);
                for (int k = 1; k < CPL; ++k) tc += cta_total(lane * CPL + k);
                const double incl = warp_scan_incl(tc, lane);
                const double T = __shfl_sync(0xffffffffu, incl, 31);
                const unsigned pos_cta = __ballot_sync(0xffffffffu, tc > 0.0);
                if (T > 0.0 && pos_cta) {
                    const double t = u_next * T;
                    // owner CTA: first with positive mass whose running total reaches t
                    unsigned m = __ballot_sync(0xffffffffu, tc > 0.0 && incl >= t);
                    const int ol = m ? __ffs(m) - 1 : 31 - __clz(pos_cta);
                    double before = __shfl_sync(0xffffffffu, incl - tc, ol);
                    int owner = ol;
                    if (CPL > 1) {
                        // the same running total through lane ol's CTAs (every lane alike)
                        int hit = -1, last = -1;
                        double c = before, hit_before = 0.0, last_before = 0.0;
                        for (int k = 0; k < CPL; ++k) {
                            const int cc = ol * CPL + k;
                            const double v = cta_total(cc);
                            const double prev = c;
                            c += v;
                            if (v > 0.0) {
                                last = cc;
                                last_before = prev;
                                if (hit < 0 && c >= t) {
                                    hit = cc;
                                    hit_before = prev;
                                }
                            }
                        }
                        owner = hit >= 0 ? hit : last;
                        before = hit >= 0 ? hit_before : last_before;
                    }
                    const double t1 = t - before;
                    // owner's chunk (its chunk sums are in the local inbox)
                    const double cv =
                        lane < nch ? (GS ? __ldcg(ginbox(cur, owner) + lane) : ib[owner * 33 + lane]) : 0.0;
                    const double ci = warp_scan_incl(cv, lane);
                    const unsigned pos_ch = __ballot_sync(0xffffffffu, cv > 0.0);
                    if (pos_ch) {  // warp-uniform; a positive total implies a positive chunk
                        m = __ballot_sync(0xffffffffu, cv > 0.0 && ci >= t1);
                        const int chunk = m ? __ffs(m) - 1 : 31 - __clz(pos_ch);
                        const double t2 = t1 - __shfl_sync(0xffffffffu, ci - cv, chunk);
                        // row inside the chunk: one read of the owner's residuals
                        float vals[kMaxPL];
                        if constexpr (GS) {
                            const float* rd = a.gs_resid + (((size_t)b * 2 + cur) * G + owner) * (size_t)Rpad +
                                              (size_t)chunk * CH;
#pragma unroll
                            for (int k = 0; k < kMaxPL; ++k) vals[k] = k < PL ? __ldcg(rd + lane * PL + k) : 0.f;
                        } else {
                            const float* rd =
                                cluster.map_shared_rank(dbuf + (size_t)cur * Rpad, owner) + (size_t)chunk * CH;
                            if (PL == 4) {  // one 16-byte read per lane
                                const float4 q4 = *reinterpret_cast<const float4*>(rd + lane * 4);
#pragma unroll
                                for (int k = 0; k < kMaxPL; ++k) vals[k] = 0.f;
                                vals[0] = q4.x; vals[1] = q4.y; vals[2] = q4.z; vals[3] = q4.w;
                            } else {
#pragma unroll
                                for (int k = 0; k < kMaxPL; ++k) vals[k] = k < PL ? rd[lane * PL + k] : 0.f;
                            }
                        }
                        double part = 0.0;
#pragma unroll
                        for (int k = 0; k < kMaxPL; ++k)
                            if (k < PL) part += (double)vals[k];
                        double c = warp_scan_incl(part, lane) - part;
                        int hit = -1, lastnz = -1;
#pragma unroll
                        for (int k = 0; k < kMaxPL; ++k) {
                            if (k >= PL) break;
                            const float v = vals[k];
                            if (v > 0.f) lastnz = k;
                            c += (double)v;
                            if (hit < 0 && v > 0.f && c >= t2) hit = k;
                        }
                        const unsigned hm = __ballot_sync(0xffffffffu, hit >= 0);
                        int local = -1;
                        if (hm) {
                            const int src = __ffs(hm) - 1;
                            local = src * PL + __shfl_sync(0xffffffffu, hit, src);
                        } else {
                            const unsigned nm = __ballot_sync(0xffffffffu, lastnz >= 0);
                            if (nm) {
                                const int src = 31 - __clz(nm);
                                local = src * PL + __shfl_sync(0xffffffffu, lastnz, src);
                            }
                        }
                        if (local >= 0) s = (int)((int64_t)owner * R + (int64_t)chunk * CH + local);
                    }
                }
            }
            if (s >= 0) {
                // warp 0 fetches the pivot's key into shared memory and starts the
                // factor row while the other warps wait at the barrier
                if (lane < LPR) {
                    float4 piece;
                    if constexpr (KRES) {
                        const int owner = (int)(s / R), lrow = (int)(s - (int64_t)owner * R);
                        piece = *cluster.map_shared_rank(
                            reinterpret_cast<const float4*>(smem + L.kres + kres_off(lrow, lane)), owner);
                    } else {
                        piece = __ldg(reinterpret_cast<const float4*>(Kb + (int64_t)s * D + lane * EPL));
                    }
                    reinterpret_cast<float4*>(ksm)[lane] = piece;
                }
                if (i <= kFsByWarp0)
                    for (int j = lane; j < i; j += 32) cp_async4(fs + j, Fb + (int64_t)j * n + s);
                cp_async_commit();
            }
            if (lane == 0) {
                imisc[3] = s;
                imisc[4] = (s < 0);
            }
        }
        __syncthreads();
        if (imisc[4]) break;
        const int s = imisc[3];

        // -- the pivot's factor row (asynchronous; first needed by the factor
        //    pass; warp 0 issued it for short rows) and the pivot key
        //    (registers of every lane) --
        if (i > kFsByWarp0) {
            for (int j = tid; j < i; j += NT) cp_async4(fs + j, Fb + (int64_t)j * n + s);
            cp_async_commit();
        }
        float xr[EPL];
        {
            const float4 raw = reinterpret_cast<const float4*>(ksm)[kl_part];
            if constexpr (sizeof(T) == 2) {
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = __bfloat1622float2(h[k]);
                    xr[2 * k] = f.x;
                    xr[2 * k + 1] = f.y;
                }
            } else {
                xr[0] = raw.x; xr[1] = raw.y; xr[2] = raw.z; xr[3] = raw.w;
            }
#pragma unroll
            for (int e = 0; e < EPL; ++e) xr[e] -= kbr[e];
        }
        if (crank == 0) {
            if (tid == 0 && a.S) a.S[b * r + i] = s;
            if (a.K_S) {
                T* dst = reinterpret_cast<T*>(a.K_S) + (b * r + i) * D;
                for (int c = tid; c < D; c += NT) dst[c] = ksm[c];
            }
        }
        // -- <k_l - kbar, k_s - kbar> for the CTA's rows --
        key_pass(xr, false, dotb);
        cp_async_wait<0>();
        __syncthreads();
        // -- pivot residual g_s (warp 0, the same on every CTA), read after the next barrier --
        if (warp == 0) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) dot = fmaf(xr[e], xr[e], dot);
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            float acc = 0.f;
            for (int j = lane; j < i; j += 32) acc = fmaf(fs[j], fs[j], acc);
            acc = warp_sum(acc);
            if (lane == 0) {
                const float gs = expf(beta * (dot - MK)) - acc;
                misc[2] = gs;
                imisc[4] = !(gs > a.eps);  // max_l h(k_l, k_l) is exp(0) = 1
            }
        }

        // -- factor pass over the CTA's rows: acc_l = sum_j F[j, l] F[j, s] --
        const int jl = (i + JG - 1) / JG, j0 = min(i, g * jl), j1 = min(i, j0 + jl);
        bool stop = false;
        for (int base = 0; base < nrows; base += TPG * VEC) {
            const int row = base + tt * VEC;
            const bool valid = row < nrows;
            float acc[VEC];
#pragma unroll
            for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
            if (valid) {
                const float* fcol = Fb + row0 + row;
                int j = j0;
                if constexpr (VEC == 4) {
                    const int cnt = j1 - j0;
#pragma unroll
                    for (int q = 0; q < INFL; ++q) {
                        if (q < cnt) cp_async16(ring4 + q * NT, fcol + (int64_t)(j0 + q) * n);
                        cp_async_commit();
                    }
                    int slot_rd = 0, slot_wr = INFL;
                    const float* src_wr = fcol + (int64_t)(j0 + INFL) * n;
                    for (int q = 0; q < cnt; ++q) {
                        if (q + INFL < cnt) cp_async16(ring4 + slot_wr * NT, src_wr);
                        cp_async_commit();
                        src_wr += n;
                        slot_wr = slot_wr + 1 == DEPTH ? 0 : slot_wr + 1;
                        cp_async_wait<INFL>();
                        const float4 v = ring4[slot_rd * NT];
                        slot_rd = slot_rd + 1 == DEPTH ? 0 : slot_rd + 1;
                        const float f = fs[j0 + q];
                        acc[0] = fmaf(v.x, f, acc[0]);
                        acc[1] = fmaf(v.y, f, acc[1]);
                        acc[2] = fmaf(v.z, f, acc[2]);
                        acc[3] = fmaf(v.w, f, acc[3]);
                    }
                    cp_async_wait<0>();
                } else {
                    for (; j + UF <= j1; j += UF) {
                        float v[UF];
#pragma unroll
                        for (int u = 0; u < UF; ++u) v[u] = ld_cg1(fcol + (int64_t)(j + u) * n);
#pragma unroll
                        for (int u = 0; u < UF; ++u) acc[0] = fmaf(v[u], fs[j + u], acc[0]);
                    }
                    for (; j < j1; ++j) acc[0] = fmaf(ld_cg1(fcol + (int64_t)j * n), fs[j], acc[0]);
                }
            }
            if (JG > 1) {
                if (g > 0) {
                    float* dst = red + ((size_t)(g - 1) * TPG + tt) * VEC;
#pragma unroll
                    for (int k = 0; k < VEC; ++k) dst[k] = acc[k];
                }
                __syncthreads();
                if (g == 0) {
                    for (int h = 0; h < JG - 1; ++h) {
                        const float* src = red + ((size_t)h * TPG + tt) * VEC;
#pragma unroll
                        for (int k = 0; k < VEC; ++k) acc[k] += src[k];
                    }
                }
            } else if (base == 0) {
                __syncthreads();  // g_s of warp 0
            }
            if (base == 0 && imisc[4]) {  // uniform: read after a barrier
                stop = true;
                break;
            }
            const float gs = misc[2];
            const float piv = sqrtf(gs);
            if (g == 0) {
                double p = 0.0;
                if (valid) {
                    float out[VEC];
#pragma unroll
                    for (int k = 0; k < VEC; ++k) {
                        const int64_t l = row0 + row + k;
                        float gl = expf(beta * (dotb[row + k] - MK)) - acc[k];
                        if (l == s) gl = gs;
                        const float f = gl / piv;
                        out[k] = f;
                        float dn = fmaxf(dcur[row + k] - f * f, 0.f);
                        if (l == s) dn = 0.f;
                        dnxt[row + k] = dn;
                        if constexpr (GS) gres(nxt)[row + k] = dn;
                        p += (double)dn;
                    }
                    float* dstF = Fb + (int64_t)i * n + row0 + row;
                    if constexpr (VEC == 4) {
                        *reinterpret_cast<float4*>(dstF) = make_float4(out[0], out[1], out[2], out[3]);
                    } else {
                        dstF[0] = out[0];
                    }
                }
                if (fused_csl) {  // the search's chunk arithmetic: four in order per lane, then the warp scan
                    const double incl = warp_scan_incl(p, lane);
                    const int ch = (base >> 7) + (tt >> 5);
                    if (lane == 31 && ch < nch) csl[ch] = incl;
                }
            }
            if (JG > 1) __syncthreads();
        }
        if (nrows == 0) {  // a CTA without rows takes the same barrier and stop test as the others
            __syncthreads();
            stop = imisc[4] != 0;
        }
        if (stop) break;
        // rows of the slice past n keep zero mass; chunks no row block reached sum to zero
        for (int row = nrows + tid; row < Rpad; row += NT) {
            dnxt[row] = 0.f;
            if constexpr (GS) gres(nxt)[row] = 0.f;
        }
        if (fused_csl) {
            const int covered = (int)(ceil_div(nrows, TPG * VEC) * (TPG * VEC / 128));
            for (int k = covered + tid; k < nch; k += NT) csl[k] = 0.0;
        }
        __syncthreads();
        publish(dnxt, nxt, fused_csl, i + 1);
    }

    // ---------------- pause at the phase end, or the effective rank and padding past it ----------------
    if (i == step_end && step_end < r && !(GS && imisc[5])) {
        // still going: keep the residual diagonal (the buffer of step i) for the next phase
        const float* dcur = dbuf + (size_t)(i & 1) * Rpad;
        float* dst = a.ph_resid + b * n + row0;
        for (int row = tid; row < nrows; row += NT) dst[row] = dcur[row];
        if (crank == 0 && tid == 0) a.act_out[atomicAdd(a.act_n_out, 1)] = (int)b;
    } else {
        const int rr = i;
        for (int j = rr; j < r; ++j) {
            float* dst = Fb + (int64_t)j * n + row0;
            for (int row = tid; row < nrows; row += NT) dst[row] = 0.f;
        }
        if (crank == 0) {
            if (tid == 0) a.rank[b] = rr;
            for (int j = rr + tid; j < r; j += NT)
                if (a.S) a.S[b * r + j] = -1;
            if (a.K_S) {
                T* dst = reinterpret_cast<T*>(a.K_S) + b * r * D;
                for (int64_t e = (int64_t)rr * D + tid; e < (int64_t)r * D; e += NT) dst[e] = T(0.f);
            }
        }
    }
    // keep this CTA's shared memory alive until every peer is done reading it
    if constexpr (!GS) cluster.sync();
}

__global__ void pivot_uniform_kernel(uint64_t seed, int64_t BH, int steps, double* u) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= BH * steps) return;
    const int64_t b = t / steps;
    const int i = (int)(t % steps);
    u[t] = pivot_uniform(seed, (uint32_t)i, (uint32_t)b);
}

template <typename E, int D, int VEC, int DEPTH, int KM, bool GS, int NTH>
cudaError_t launch_select_t(const SelectArgs& a, size_t smem, cudaStream_t stream) {
    auto kern = rpc_select_kernel<E, D, VEC, DEPTH, KM, GS, NTH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (!GS && a.G > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.grid_ctas > 0 ? a.grid_ctas : a.BH * a.G));
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (GS) {
        // every CTA of the grid is co-resident, or the launch fails
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = a.G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// Clusters of G CTAs that fit at once (cluster mode) or CTAs that fit at
// once on the whole GPU (global-sync mode).
template <typename E, int D, int VEC, int DEPTH, int KM, bool GS, int NTH>
int fit_t(int G, size_t smem) {
    auto kern = rpc_select_kernel<E, D, VEC, DEPTH, KM, GS, NTH>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (GS) {
        int per_sm = 0, dev = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTH, smem) != cudaSuccess ||
            cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        return per_sm * sms;
    }
    if (G > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return nc;
}

template <typename E, int VEC, int DEPTH, int KM, bool GS, int NTH = 512>
int dispatch_d(int d, const SelectArgs* a, size_t smem, cudaStream_t stream, int G_query, cudaError_t* err) {
    switch (d) {
        case 32:
            if (a) { *err = launch_select_t<E, 32, VEC, DEPTH, KM, GS, NTH>(*a, smem, stream); return 0; }
            return fit_t<E, 32, VEC, DEPTH, KM, GS, NTH>(G_query, smem);
        case 64:
            if (a) { *err = launch_select_t<E, 64, VEC, DEPTH, KM, GS, NTH>(*a, smem, stream); return 0; }
            return fit_t<E, 64, VEC, DEPTH, KM, GS, NTH>(G_query, smem);
        case 128:
            if (a) { *err = launch_select_t<E, 128, VEC, DEPTH, KM, GS, NTH>(*a, smem, stream); return 0; }
            return fit_t<E, 128, VEC, DEPTH, KM, GS, NTH>(G_query, smem);
    }
    if (err) *err = cudaErrorInvalidValue;
    return 0;
}

// Kernel variants: the vectorised path with ring depth 24/16/12/6 (12 also
// with resident keys); the scalar path (n not a multiple of 4) with depth 6.
// The global-sync mode exists for the vectorised streamed-key variants.
struct Variant {
    int depth;
    int km;        // key mode: 0 streamed, 1 resident
    int nt = 512;  // threads per CTA (256 only for resident keys on CUDA cores)
};

template <typename E>
int dispatch_e(const Variant& v, int vec, int d, bool gs, const SelectArgs* a, size_t smem, cudaStream_t stream,
               int G_query, cudaError_t* err) {
    if (gs) {
        if (vec != 4 || v.km) {
            if (err) *err = cudaErrorInvalidValue;
            return 0;
        }
        switch (v.depth) {
            case 24: return dispatch_d<E, 4, 24, 0, true>(d, a, smem, stream, G_query, err);
            case 16: return dispatch_d<E, 4, 16, 0, true>(d, a, smem, stream, G_query, err);
            case 12: return dispatch_d<E, 4, 12, 0, true>(d, a, smem, stream, G_query, err);
        }
        return dispatch_d<E, 4, 6, 0, true>(d, a, smem, stream, G_query, err);
    }
    if (vec != 4) return dispatch_d<E, 1, 6, 0, false>(d, a, smem, stream, G_query, err);
    if (v.km == 1) {
        if (v.nt == 256) return dispatch_d<E, 4, 12, 1, false, 256>(d, a, smem, stream, G_query, err);
        return dispatch_d<E, 4, 12, 1, false>(d, a, smem, stream, G_query, err);
    }
    switch (v.depth) {
        case 24: return dispatch_d<E, 4, 24, 0, false>(d, a, smem, stream, G_query, err);
        case 16: return dispatch_d<E, 4, 16, 0, false>(d, a, smem, stream, G_query, err);
        case 12: return dispatch_d<E, 4, 12, 0, false>(d, a, smem, stream, G_query, err);
    }
    return dispatch_d<E, 4, 6, 0, false>(d, a, smem, stream, G_query, err);
}

int dispatch(const Variant& v, int dtype, int vec, int d, bool gs, const SelectArgs* a, size_t smem,
             cudaStream_t stream, int G_query, cudaError_t* err) {
    return dtype == 1 ? dispatch_e<BF16>(v, vec, d, gs, a, smem, stream, G_query, err)
                      : dispatch_e<F32>(v, vec, d, gs, a, smem, stream, G_query, err);
}

int g_cluster_override = 0;
int g_kernel_override = 0;
int g_phase_steps = 0;  // 0 automatic, > 0 fixed phase length, < 0 one launch
thread_local int g_last_cluster = 0;
thread_local int g_last_kernel = 0;
thread_local int g_last_threads = 0;
thread_local int g_last_phases = 0;

}  // namespace

constexpr int kMaxRowsPerCta = 16384;

// Memo of the automatic cluster size per device and shape (the occupancy
// queries cost host time on every launch otherwise).
bool ClusterKey::operator<(const ClusterKey& o) const {
    return std::tie(dev, kernel, n, BH, r, d, dtype) < std::tie(o.dev, o.kernel, o.n, o.BH, o.r, o.d, o.dtype);
}

static std::mutex g_cluster_mu;
static std::map<ClusterKey, int> g_cluster_memo;

int cached_cluster_lookup(const ClusterKey& key) {
    std::lock_guard<std::mutex> lock(g_cluster_mu);
    const auto it = g_cluster_memo.find(key);
    return it == g_cluster_memo.end() ? 0 : it->second;
}

void cached_cluster_store(const ClusterKey& key, int G) {
    std::lock_guard<std::mutex> lock(g_cluster_mu);
    g_cluster_memo[key] = G;
}

// Cluster size for one select launch.  Candidates are G in {1, 2, 4, 8, 16}
// with at most kMaxRowsPerCta rows per CTA and at least min_rows (unless G = 1);
// fit(G) is the number of clusters of G CTAs that fit on the GPU at once
// (0 = not schedulable).  The cost of G is the rows one CTA streams times
// the waves of clusters, ceil(BH / fit) * ceil(n / G): a 16-CTA cluster must
// sit inside one GPC, so fewer of them fit than the SM count suggests.
int choose_cluster_rows(int64_t n, int64_t BH, int (*fit)(int G, void* ctx), void* ctx, double* cost_out,
                        int min_rows) {
    int best = 0;
    double best_cost = 0.0;
    for (int g = 1; g <= 16; g *= 2) {
        const int64_t rows = ceil_div(n, g);
        if (rows > kMaxRowsPerCta) continue;
        if (g > 1 && n / g < min_rows) break;
        const int f = fit(g, ctx);
        if (f <= 0) continue;
        const double cost = (double)ceil_div(BH, f) * (double)rows;
        if (best == 0 || cost < best_cost * 0.999) {
            best = g;
            best_cost = cost;
        }
    }
    if (cost_out) *cost_out = best_cost;
    return best;
}

// Workspace of the global-sync mode (G <= kGsMaxCtas CTAs per instance) and
// of phased launches.  ctl holds [count 0][barrier counter per instance][count 1]
// so that one memset clears a launch's barriers and its output count.
struct SelectWs {
    double* inbox;
    float* resid;
    unsigned* ctl;
    float* mk;
    float* ph_resid;
    float* ph_mk;
    int* act;  // two lists of BH instance indices
    size_t used;
    bool fits;
};
static SelectWs carve_select_ws(void* ws, size_t bytes, int64_t BH, int64_t n) {
    Carve cv(ws, bytes);
    SelectWs w{};
    w.inbox = static_cast<double*>(cv.take(sizeof(double) * BH * 2 * kGsMaxCtas * 33));
    w.resid = static_cast<float*>(cv.take(sizeof(float) * BH * 2 * (n + (int64_t)kGsMaxCtas * 520)));  // G Rpad <= n + G (4 + 511)
    w.ctl = static_cast<unsigned*>(cv.take(sizeof(unsigned) * (BH + 2)));
    w.mk = static_cast<float*>(cv.take(sizeof(float) * BH * kGsMaxCtas));
    w.ph_resid = static_cast<float*>(cv.take(sizeof(float) * BH * n));
    w.ph_mk = static_cast<float*>(cv.take(sizeof(float) * BH));
    w.act = static_cast<int*>(cv.take(sizeof(int) * 2 * BH));
    w.used = cv.used;
    w.fits = cv.fits();
    return w;
}
size_t select_workspace_bytes(int64_t BH, int64_t n) { return carve_select_ws(nullptr, 0, BH, n).used + 256; }

int read_select_gs_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_select_gs_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_select_gs_status, &z, sizeof(int));
    }
    return v;
}

int select_cluster_override(int G) {
    if (G < 0) return g_cluster_override;
    g_cluster_override = G;
    return G;
}
int last_select_cluster() { return g_last_cluster; }
int select_kernel_override(int k) {
    if (k < 0) return g_kernel_override;
    g_kernel_override = k;
    return k;
}
// test hook of the global-sync barrier (wildcat_test_force_select_timeout)
static unsigned long long g_force_select_timeout_ns = 0;
void set_select_force_timeout(unsigned long long ns) { g_force_select_timeout_ns = ns; }
unsigned long long select_force_timeout_ns() { return g_force_select_timeout_ns; }
int last_select_kernel() { return g_last_kernel; }
int last_select_threads() { return g_last_threads; }
int select_phase_steps_override(int k, bool set) {
    if (set) g_phase_steps = k;
    return g_phase_steps;
}
int last_select_phases() { return g_last_phases; }

static void plan(int64_t n, int r, int d, int dtype, int G, int vec, bool gs, SelectArgs* a, size_t* smem,
                 Variant* v, int nt = 512) {
    const SelectShape sh(n, G, nt, vec);
    const int R = sh.R, JG = sh.JG, PL = sh.PL, Rpad = sh.Rpad;
    a->G = G;
    a->R = R;
    a->JG = JG;
    a->PL = PL;
    auto bytes = [&](int depth, int km) {
        const size_t kb = km ? (size_t)R * d * (dtype == 1 ? 2 : 4) : 0;
        return SmemLayout(Rpad, r, d, JG, nt, vec, G, depth, kb, gs).total;
    };
    if (gs) {
        *v = {6, 0};  // streamed keys only
        for (int depth : {24, 16, 12})
            if (bytes(depth, 0) <= kSmemCap) {
                *v = {depth, 0};
                break;
            }
    } else if (vec != 4) {
        *v = {6, 0};
    } else if (bytes(12, 1) <= kSmemCap) {
        *v = {12, 1};  // keys stay in shared memory: the per-step key pass reads no global memory
    } else {
        *v = {6, 0};
        for (int depth : {24, 16, 12})
            if (bytes(depth, 0) <= kSmemCap) {
                *v = {depth, 0};
                break;
            }
    }
    if (nt != 512) {
        // the 256-thread form exists for resident keys on CUDA cores only
        *v = (!gs && vec == 4 && bytes(12, 1) <= kSmemCap) ? Variant{12, 1, nt} : Variant{0, -1, nt};
        *smem = v->km < 0 ? kSmemCap + 1 : bytes(12, 1);
        return;
    }
    *smem = bytes(v->depth, v->km);
}

struct ClusterCtx {
    const SelectRequest* q;
    const SelectArgs* a;
    int vec;
    cudaStream_t stream;
    int nt = 512;
};

// Clusters of g CTAs that fit at once for this request's kernel variant.
static int cluster_fit(int g, void* p) {
    const ClusterCtx& c = *static_cast<const ClusterCtx*>(p);
    SelectArgs t = *c.a;
    Variant v{};
    size_t sm = 0;
    plan(c.q->n, c.q->r, c.q->d, c.q->dtype, g, c.vec, false, &t, &sm, &v, c.nt);
    if (sm > kSmemCap) return 0;
    return dispatch(v, c.q->dtype, c.vec, c.q->d, false, nullptr, sm, c.stream, g, nullptr);
}

// Two 256-thread CTAs per SM overlap each other's barriers and searches but
// share the SM's issue slots and bandwidth: their rows per CTA count 1.3x.
constexpr double kHalfCtaCost = 1.3;

// Phases: the factorisation of a long coreset runs as launches of `len`
// steps.  The first is the ordinary launch; after it the instances still going
// (the others truncated) continue in global-sync launches of the whole GPU,
// each with about SMs / (instances left) CTAs, so that the longest factors no
// longer run on the few CTAs the first launch gave them.
constexpr int kPhaseMinRank = 512;
constexpr int kPhaseSteps = 64;  // c. 50 us per boundary against the rebalancing it allows
struct PhasePlan {
    int len = 0;
    int Gmin = 0;
    int P = 0;
    Variant var{};
    size_t smem = 0;
    SelectArgs ra{};
};
static bool plan_phases(const SelectRequest& q, const SelectArgs& a, int vec, int sms, cudaStream_t st,
                        PhasePlan* pp) {
    int len = g_phase_steps;
    if (len == 0) len = q.r >= kPhaseMinRank ? kPhaseSteps : 0;
    if (len <= 0 || len >= q.r || vec != 4 || q.BH > sms) return false;
    // the least G a resumed launch gives an instance: all BH still going
    const int Gmin = (int)std::min<int64_t>(std::min<int64_t>(32, sms / q.BH), std::max<int64_t>(1, q.n / 256));
    if (ceil_div(q.n, Gmin) > kMaxRowsPerCta) return false;
    SelectArgs ra = a;
    Variant var{};
    size_t smem = 0;
    plan(q.n, q.r, q.d, q.dtype, Gmin, vec, true, &ra, &smem, &var);
    if (smem > kSmemCap) return false;
    // the kernel may give an instance any G in [Gmin, kGsMaxCtas]: room for the largest layout
    for (int G = Gmin; G <= kGsMaxCtas; ++G) {
        const SelectShape sh(q.n, G, 512, vec);
        smem = std::max(smem, SmemLayout(sh.Rpad, q.r, q.d, sh.JG, 512, vec, G, var.depth, 0, true).total);
    }
    if (smem > kSmemCap) return false;
    int P = dispatch(var, q.dtype, vec, q.d, true, nullptr, smem, st, Gmin, nullptr);
    P = std::min(P, sms);
    if (P < q.BH * Gmin) return false;
    pp->len = len;
    pp->Gmin = Gmin;
    pp->P = P;
    pp->var = var;
    pp->smem = smem;
    pp->ra = ra;
    return true;
}

Status launch_select(const SelectRequest& q, cudaStream_t stream) {
    const int vec = (q.n % 4 == 0) ? 4 : 1;
    SelectArgs a{};
    a.K = q.K;
    a.BH = q.BH;
    a.n = q.n;
    a.beta = q.beta;
    a.r = q.r;
    a.seed = q.seed;
    a.inst0 = q.inst0;
    a.kbar = q.kbar;
    a.kbar_div = q.kbar_div > 0 ? q.kbar_div : 1;
    a.eps = q.eps;
    a.S_fixed = q.S_fixed;
    a.S = q.S;
    a.F = q.F;
    a.rank = q.rank;
    a.K_S = q.K_S;
    a.step0 = 0;
    a.step_end = q.r;
    g_last_phases = 1;

    size_t smem = 0;
    Variant var{};
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    ClusterCtx ctx{&q, &a, vec, stream};

    const bool ws_ok = q.ws && q.ws_bytes >= select_workspace_bytes(q.BH, q.n) && vec == 4 &&
                       (reinterpret_cast<uintptr_t>(q.ws) & 255u) == 0;
    const SelectWs w = ws_ok ? carve_select_ws(q.ws, q.ws_bytes, q.BH, q.n) : SelectWs{};
    PhasePlan pp;
    const bool phased = ws_ok && w.fits && plan_phases(q, a, vec, sms, stream, &pp);
    if (phased) {
        a.step_end = pp.len;
        a.ph_resid = w.ph_resid;
        a.ph_mk = w.ph_mk;
        a.act_out = w.act;
        a.act_n_out = reinterpret_cast<int*>(w.ctl);
        // count 0 and the barrier counters of the first launch
        const cudaError_t err = cudaMemsetAsync(w.ctl, 0, sizeof(unsigned) * (q.BH + 1), stream);
        if (err != cudaSuccess) return Status::cuda(err, "select: phase counters");
    }
    // the launches after the first one (global sync over the whole GPU)
    auto resume = [&]() -> Status {
        if (!phased) return Status::ok();
        const int nph = (int)ceil_div(q.r, pp.len);
        for (int p = 1; p < nph; ++p) {
            SelectArgs ra = pp.ra;
            ra.gs_inbox = w.inbox;
            ra.gs_resid = w.resid;
            ra.gs_mk = w.mk;
            ra.gs_bar = w.ctl + 1;
            ra.gs = 1;
            ra.gs_force_ns = select_force_timeout_ns();
            ra.step0 = p * pp.len;
            ra.step_end = std::min(q.r, (p + 1) * pp.len);
            ra.ph_resid = w.ph_resid;
            ra.ph_mk = w.ph_mk;
            ra.act_in = w.act + (size_t)((p - 1) & 1) * q.BH;
            ra.act_n_in = reinterpret_cast<int*>(w.ctl + (((p - 1) & 1) ? q.BH + 1 : 0));
            ra.act_out = w.act + (size_t)(p & 1) * q.BH;
            ra.act_n_out = reinterpret_cast<int*>(w.ctl + ((p & 1) ? q.BH + 1 : 0));
            ra.grid_ctas = pp.P;
            // this launch's barrier counters and output count ([count 0][barriers][count 1])
            cudaError_t err = cudaMemsetAsync(w.ctl + ((p & 1) ? 1 : 0), 0, sizeof(unsigned) * (q.BH + 1), stream);
            if (err == cudaSuccess) dispatch(pp.var, q.dtype, vec, q.d, true, &ra, pp.smem, stream, pp.Gmin, &err);
            if (err == cudaSuccess) err = cudaGetLastError();
            if (err != cudaSuccess) return Status::cuda(err, "select (resumed phase) launch");
        }
        g_last_phases = nph;
        return Status::ok();
    };

    // Global-sync mode: given a workspace and few instances, more CTAs per
    // instance than clusters allow (all co-resident by a cooperative launch).
    if (ws_ok && g_kernel_override != 1 && g_cluster_override <= 0) {
        const ClusterKey gkey{dev, g_kernel_override == 3 ? 4 : 3, q.n, q.BH, q.r, q.d, q.dtype};
        int Gg = cached_cluster_lookup(gkey);
        if (Gg == 0) {
            Gg = -1;
            const int cand = (int)std::min<int64_t>(32, sms / std::max<int64_t>(1, q.BH));
            if (cand >= 2 && q.n / cand >= 512 && ceil_div(q.n, cand) <= kMaxRowsPerCta) {
                SelectArgs t = a;
                Variant v{};
                size_t sm = 0;
                plan(q.n, q.r, q.d, q.dtype, cand, vec, true, &t, &sm, &v);
                const int fit = sm <= kSmemCap ? dispatch(v, q.dtype, vec, q.d, true, nullptr, sm, stream, cand, nullptr)
                                               : 0;
                if (fit >= q.BH * cand) {
                    double cc = 0.0;
                    const int Gc = choose_cluster_rows(q.n, q.BH, cluster_fit, &ctx, &cc, 512);
                    // the global barrier and L2 round trips cost more per step than a cluster's
                    const double cg = 1.15 * (double)ceil_div(q.n, cand);
                    if (g_kernel_override == 3 || Gc <= 0 || cg < cc) Gg = cand;
                }
            }
            cached_cluster_store(gkey, Gg);
        }
        if (Gg > 0) {
            plan(q.n, q.r, q.d, q.dtype, Gg, vec, true, &a, &smem, &var);
            if (!w.fits) return Status::fail(4, "select: workspace too small");
            a.gs_inbox = w.inbox;
            a.gs_resid = w.resid;
            a.gs_bar = w.ctl + 1;
            a.gs_mk = w.mk;
            a.gs = 1;
            a.gs_force_ns = select_force_timeout_ns();
            cudaError_t err = phased ? cudaSuccess : cudaMemsetAsync(w.ctl + 1, 0, sizeof(unsigned) * q.BH, stream);
            if (err == cudaSuccess) dispatch(var, q.dtype, vec, q.d, true, &a, smem, stream, Gg, &err);
            if (err == cudaSuccess) err = cudaGetLastError();
            if (err != cudaSuccess) return Status::cuda(err, "select (global sync) launch");
            g_last_cluster = Gg;
            g_last_kernel = 3;
            g_last_threads = 512;
            return resume();
        }
    }

    int G = g_cluster_override;
    int nt = 512;
    if (G <= 0) {
        // the cluster size (and CTA width) with the least work per CTA times waves of clusters
        const ClusterKey key{dev, 1, q.n, q.BH, q.r, q.d, q.dtype};
        const int memo = cached_cluster_lookup(key);
        if (memo > 0) {
            G = memo & 0xff;
            nt = (memo & 0x100) ? 256 : 512;
        } else {
            double c512 = 0.0, c256 = 0.0;
            G = choose_cluster_rows(q.n, q.BH, cluster_fit, &ctx, &c512, 512);
            if (g_kernel_override != 4) {
                ClusterCtx ctx256 = ctx;
                ctx256.nt = 256;
                const int G256 = choose_cluster_rows(q.n, q.BH, cluster_fit, &ctx256, &c256, 256);
                // only in one wave: with waves of clusters the rows-per-CTA model
                // misjudged it (128 instances of 4096 keys ran 1.7x slower)
                const bool one_wave = G256 > 0 && cluster_fit(G256, &ctx256) >= q.BH;
                if (one_wave && (G <= 0 || kHalfCtaCost * c256 < c512)) {
                    G = G256;
                    nt = 256;
                }
            }
            if (G > 0) cached_cluster_store(key, G | (nt == 256 ? 0x100 : 0));
        }
        if (G <= 0) return Status::fail(2, "select: no schedulable cluster shape (n / 16 above 16384 rows?)");
    } else if (ceil_div(q.n, G) > kMaxRowsPerCta) {
        return Status::fail(2, "select: n / G exceeds the per-CTA row limit (16384)");
    }
    plan(q.n, q.r, q.d, q.dtype, G, vec, false, &a, &smem, &var, nt);
    if (smem > kSmemCap) return Status::fail(2, "select: shared memory plan exceeds 227 KB");
    cudaError_t err = cudaSuccess;
    dispatch(var, q.dtype, vec, q.d, false, &a, smem, stream, G, &err);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return Status::cuda(err, "select launch");
    g_last_cluster = G;
    g_last_kernel = var.km == 2 ? 4 : 1;
    g_last_threads = nt;
    return resume();
}

Status launch_pivot_uniforms(uint64_t seed, int64_t BH, int steps, double* u, cudaStream_t stream) {
    const int64_t total = BH * steps;
    if (total == 0) return Status::ok();
    pivot_uniform_kernel<<<(unsigned)ceil_div(total, 256), 256, 0, stream>>>(seed, BH, steps, u);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return Status::cuda(err, "pivot uniforms launch");
    return Status::ok();
}

}  // namespace wildcat
