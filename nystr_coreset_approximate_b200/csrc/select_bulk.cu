// select_bulk.cu -- RPCholesky coreset selection, bulk-copy streaming kernel (sm_100a).
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2
// (randomly pivoted Cholesky; Alg. 1 RPNys).  The arithmetic is that of
// select.cu: one thread-block cluster of G CTAs per instance, CTA c owns key
// rows [c R, c R + R), the residual diagonal lives in shared memory, every
// CTA runs the same pivot search, one cluster barrier per step.  What
// differs is how the per-step streams reach the CTA:
//
//  * K rows and the factor prefix F[0..i-2, rows] are moved by the copy
//    engine (cp.async.bulk, one instruction per contiguous run, completion
//    counted in bytes on an mbarrier) into a ring of NS stages of 32 KB.
//    Consumers release a stage with one mbarrier arrival per warp; thread 0
//    refills released stages without blocking.
//  * None of the streamed data depends on the pivot (only the arithmetic
//    does), so the stream runs on across steps: the first stages of step
//    i+1 are in flight while step i finishes, the cluster synchronises and
//    the next pivot is drawn.  Tiles of step i read columns <= i-2 only,
//    written (and fenced for the async proxy) two steps earlier.
//  * Column i-1 of the factor stays in the registers of the thread that
//    wrote it, so step i never waits for step i-1's stores.
//  * The chunk sums the pivot search needs are formed in the epilogue that
//    writes the new residual, and the search itself uses warp scans.
//
// Every mbarrier wait is bounded (2 s).  A CTA whose wait expires records
// WILDCAT_ERR_TIMEOUT, stops waiting, and announces the abort to its
// cluster with its chunk sums; the next pivot search of every CTA sees it
// and all stop at the same step.  Before exiting, thread 0 waits (bounded)
// for every copy it issued.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "philox.cuh"
#include "tc_common.cuh"

namespace cg = cooperative_groups;

namespace wildcat {

__device__ int g_select_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

namespace {

using tc::globaltimer;
using tc::kWaitLimitNs;
using tc::smem_u32;

constexpr int kBT = 512, kBW = kBT / 32;
constexpr int kStageBytes = 32 * 1024;
constexpr int kChunk = 128;          // rows per search chunk: 32 lanes x 4 rows
constexpr int kNchMax = 64;          // search chunks per CTA (R <= 8192)
constexpr int kInbox = kNchMax + 2;  // per source CTA: chunk sums, total, abort flag
constexpr int kMaxQPT = 4;           // row quads per thread in the factor pass
constexpr int kMaxStages = 8;
constexpr size_t kSmemCap = 226 * 1024;  // 227 KB per block, less room for the static shared array

unsigned long long g_force_select_timeout_ns = 0;

struct BulkArgs {
    const void* K;
    int64_t BH, n;
    float beta;
    int r;
    uint64_t seed;
    int64_t inst0;
    const float* kbar;
    int kbar_div;
    float eps;
    const int32_t* S_fixed;
    int32_t* S;
    float* F;
    int32_t* rank;
    void* K_S;
    int G, R;
    int NS;   // ring stages
    int CPT;  // factor columns per stage
    int NKT;  // key tiles per pass (0 with resident keys)
    int KTR;  // key rows per stage
    int JG, TPG, QPT;
    unsigned long long force_timeout_ns;  // test hook: one bounded wait on a barrier nothing completes
};

struct BulkLayout {
    size_t ring, kres, dbuf, dotb, red, inbox, csl, fs, bars, misc, total;
    __host__ __device__ BulkLayout(int R, int r, int rowbytes, int NS, int G, int JG, int TPG, bool kres_on) {
        const int64_t Rpad = round_up(R, kChunk);
        size_t o = 0;
        ring = o;  o += (size_t)NS * kStageBytes;
        kres = o;  o += kres_on ? (size_t)round_up((int64_t)R * rowbytes, 16) : 0;
        dbuf = o;  o += 2 * (size_t)Rpad * sizeof(float);
        dotb = o;  o += (size_t)Rpad * sizeof(float);
        red = o;   o += (size_t)(JG - 1) * TPG * 16;
        inbox = o; o += 2 * (size_t)G * kInbox * sizeof(double);
        csl = o;   o += kNchMax * sizeof(double);
        fs = o;    o += (size_t)round_up((int64_t)r * 4, 16);
        bars = o;  o += (2 * (size_t)NS + 2) * 8;
        misc = o;  o += 64;
        total = round_up((int64_t)o, 128);
    }
};

// ---- PTX helpers ----
__device__ __forceinline__ void mbar_arrive(uint64_t* m) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(m)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* m, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(m)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* m, unsigned parity) {
    unsigned done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(smem_u32(m)), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* m) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(m))
        : "memory");
}
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Inclusive fp64 warp scan (Hillis-Steele); identical on every CTA.
__device__ __forceinline__ double warp_scan_incl(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Sum of four residuals in a fixed order (the epilogue and the search use it alike).
__device__ __forceinline__ double quad_sum(float a, float b, float c, float d) {
    return (((double)a + (double)b) + (double)c) + (double)d;
}

template <typename T, int EPL>
__device__ __forceinline__ void widen(const float4& raw, float (&v)[EPL]) {
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
}

// Warp-cooperative dot products of key rows with x (or |k|^2 when SELF):
// LPR lanes share a row, each widening one 16-byte piece; four rows per lane
// per iteration.  src points at row rb of the CTA; results go to out[rb + row].
template <typename T, int D, bool SELF, bool KBAR>
__device__ __forceinline__ void key_rows(const T* src, int rb, int nr, const float* x, const float* kbr,
                                         float* out, int warp, int lane) {
    constexpr int EPL = 16 / (int)sizeof(T), LPR = D / EPL, RPW = 32 / LPR, ROWS_PASS = kBW * RPW;
    const int kl_row = lane / LPR, kl_part = lane % LPR;
    for (int base = warp * RPW; base < nr; base += 4 * ROWS_PASS) {
        float part[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int row = base + u * ROWS_PASS + kl_row;
            part[u] = 0.f;
            if (row < nr) {
                const float4 raw = *reinterpret_cast<const float4*>(src + (size_t)row * D + kl_part * EPL);
                float v[EPL];
                widen<T, EPL>(raw, v);
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    if constexpr (KBAR) v[e] -= kbr[e];
                    part[u] = fmaf(v[e], SELF ? v[e] : x[e], part[u]);
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
                const int row = base + u * ROWS_PASS + kl_row;
                if (row < nr) out[rb + row] = part[u];
            }
        }
    }
}

template <typename E, int D, bool KRES, bool KBAR>
__global__ void __launch_bounds__(kBT, 1) rpc_select_bulk_kernel(const BulkArgs a) {
    // Launched with a cluster dimension of a.G (one cluster per instance).
    using T = typename E::T;
    constexpr int EPL = 16 / (int)sizeof(T);  // key elements per 16-byte piece
    constexpr int LPR = D / EPL;              // lanes per key row
    constexpr int ROWB = D * (int)sizeof(T);
    constexpr unsigned FULL = 0xffffffffu;
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int64_t b = blockIdx.x / a.G;
    if (b >= a.BH) return;  // whole clusters only: G divides gridDim.x

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = a.R, r = a.r, G = a.G, NS = a.NS, CPT = a.CPT, NKT = KRES ? 0 : a.NKT, KTR = a.KTR;
    const int JG = a.JG, TPG = a.TPG, QPT = a.QPT;
    const int64_t n = a.n;
    const int64_t row0 = (int64_t)crank * R;
    const int nrows = row0 < n ? (int)std::min<int64_t>(R, n - row0) : 0;
    const int Rpad = (int)round_up(R, kChunk), nch = Rpad / kChunk;

    extern __shared__ __align__(128) unsigned char smem[];
    const BulkLayout L(R, r, ROWB, NS, G, JG, TPG, KRES);
    unsigned char* ring = smem + L.ring;
    const T* kres = reinterpret_cast<const T*>(smem + L.kres);
    float* dbuf = reinterpret_cast<float*>(smem + L.dbuf);
    float* dotb = reinterpret_cast<float*>(smem + L.dotb);
    float4* red = reinterpret_cast<float4*>(smem + L.red);
    double* inbox = reinterpret_cast<double*>(smem + L.inbox);
    double* csl = reinterpret_cast<double*>(smem + L.csl);
    float* fs = reinterpret_cast<float*>(smem + L.fs);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* never = empty + NS;  // test hook: nothing ever arrives here
    float* misc = reinterpret_cast<float*>(smem + L.misc);
    volatile int* imisc = reinterpret_cast<volatile int*>(misc);
    // misc[0] local max |k|^2, misc[1] M_K, misc[2] g_s; imisc[3] s, imisc[4] stop, imisc[5] abort

    const T* Kb = reinterpret_cast<const T*>(a.K) + b * n * D;
    float* Fb = a.F + b * (int64_t)r * n;
    const int kl_part = lane % LPR;
    float kbr[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) kbr[e] = KBAR ? a.kbar[(b / a.kbar_div) * D + kl_part * EPL + e] : 0.f;

    // factor-pass mapping: group g of TPG threads takes every JG-th column of
    // a stage; thread tt of a group owns row quads tt + k TPG (k < QPT)
    const int g = tid / TPG, tt = tid % TPG;

    // ---------------- the ring: producer (thread 0) and consumers ----------------
    // Tiles of step i: NKT key tiles, then ceil((i-1)/CPT) factor tiles
    // (columns 0..i-2); step -1 is the prologue's key pass.
    auto ntiles = [&](int step) -> int { return NKT + (step >= 1 ? (step - 1 + CPT - 1) / CPT : 0); };
    // The producer is warp 0, converged: every lane keeps the same cursor and
    // takes the same decisions (a lone producer lane beside 31 spinning lanes
    // could wait long for the scheduler); lane 0 arms the stage's barrier and
    // the lanes share the copies.  Slots and barrier phases advance
    // incrementally on both sides.
    int p_step = -1, p_pos = 0;  // producer cursor (warp 0)
    long long tiss = 0;          // tiles issued (warp 0)
    int p_slot = 0;              // stage of tile tiss (warp 0)
    unsigned p_par = 1;          // empty-barrier parity to test before reusing p_slot (warp 0)
    long long tcons = 0;         // tiles consumed (uniform)
    int c_slot = 0;              // stage of tile tcons (uniform)
    unsigned c_par = 0;          // full-barrier parity of tile tcons (uniform)
    int done_step = 0;           // epilogues completed (uniform)
    auto issue = [&](int step, int pos, int slot) {  // warp 0, converged
        uint64_t* fb = full + slot;
        unsigned char* dst = ring + (size_t)slot * kStageBytes;
        if (pos < NKT) {
            const int r0 = pos * KTR, nr = std::min(KTR, nrows - r0);
            const unsigned bytes = nr > 0 ? (unsigned)(nr * ROWB) : 0u;
            if (lane == 0) {
                mbar_arrive_tx(fb, bytes);
                if (bytes) bulk_g2s(dst, Kb + (row0 + r0) * D, bytes, fb);
            }
        } else {
            const int c0 = (pos - NKT) * CPT, nc = std::min(CPT, step - 1 - c0);
            const unsigned cb = (unsigned)nrows * 4u;
            if (lane == 0) mbar_arrive_tx(fb, cb * (unsigned)nc);
            __syncwarp();
            if (cb && (int64_t)R == n) {
                // one CTA per instance: the stage's columns are one contiguous run of F
                if (lane == 0) bulk_g2s(dst, Fb + (int64_t)c0 * n, cb * (unsigned)nc, fb);
            } else if (cb) {
                for (int cc = lane; cc < nc; cc += 32)
                    bulk_g2s(dst + (size_t)cc * R * 4, Fb + (int64_t)(c0 + cc) * n + row0, cb, fb);
            }
        }
        __syncwarp();
    };
    // Issue every tile whose stage is free and whose columns exist; never blocks.
    auto refill = [&]() {  // warp 0, converged
        while (p_step < r && p_step <= done_step + 1) {
            if (p_pos >= ntiles(p_step)) {
                ++p_step;
                p_pos = 0;
                continue;
            }
            if (tiss >= NS) {
                const bool freed = __shfl_sync(FULL, (int)mbar_test(empty + p_slot, p_par), 0) != 0;
                if (!freed) return;
            }
            issue(p_step, p_pos, p_slot);
            ++tiss;
            ++p_pos;
            if (++p_slot == NS) {
                p_slot = 0;
                p_par ^= 1u;
            }
        }
    };
    auto set_abort = [&]() {
        imisc[5] = 1;
        atomicExch(&g_select_status, 5);
    };
    // Wait for the next tile; returns its stage.
    auto acquire = [&]() -> const unsigned char* {
        if (warp == 0 && !imisc[5] && tiss <= tcons) {
            // the tile is not issued yet: its stage frees when the slowest warp is done
            const unsigned long long t0 = globaltimer();
            for (;;) {
                refill();
                if (tiss > tcons) break;
                if (__shfl_sync(FULL, (int)(globaltimer() - t0 > kWaitLimitNs), 0)) {
                    if (lane == 0) set_abort();
                    break;
                }
            }
            __syncwarp();
        }
        if (!imisc[5] && !tc::mbar_wait(full + c_slot, c_par)) set_abort();
        return ring + (size_t)c_slot * kStageBytes;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + c_slot);
        ++tcons;
        if (++c_slot == NS) {
            c_slot = 0;
            c_par ^= 1u;
        }
        if (warp == 0) refill();
    };

    // Chunk sums + abort flag pushed into every peer's inbox[par][crank]; the
    // cluster barrier is split so that thread 0 refills the ring and warp 0
    // draws the next uniform while the cluster arrives.
    double u_next = 0.0;  // warp 0: uniform of the next step
    auto publish = [&](int par, int next_step) {
        if (warp == 0) {
            if (a.force_timeout_ns && next_step == 2 && lane == 0) {
                // test hook: a wait that nothing completes, bounded like every other
                if (!tc::mbar_wait(never, 0, a.force_timeout_ns)) set_abort();
            }
            __syncwarp();
            const double v0 = 2 * lane < nch ? csl[2 * lane] : 0.0;
            const double v1 = 2 * lane + 1 < nch ? csl[2 * lane + 1] : 0.0;
            const double tot = __shfl_sync(FULL, warp_scan_incl(v0 + v1, lane), 31);
            const double ab = imisc[5] ? 1.0 : 0.0;
            for (int c = 0; c < G; ++c) {
                double* dst = cluster.map_shared_rank(inbox + ((size_t)par * G + crank) * kInbox, c);
                if (2 * lane < nch) dst[2 * lane] = v0;
                if (2 * lane + 1 < nch) dst[2 * lane + 1] = v1;
                if (lane == 0) {
                    dst[kNchMax] = tot;
                    dst[kNchMax + 1] = ab;
                }
            }
        }
        cluster.barrier_arrive();
        if (warp == 0) {
            refill();
            u_next = pivot_uniform(a.seed, (uint32_t)next_step, (uint32_t)(a.inst0 + b));
        }
        cluster.barrier_wait();
    };

    // ---------------- prologue ----------------
    if (tid == 0) {
        for (int k = 0; k < NS; ++k) {
            tc::mbar_init(full + k, 1);
            tc::mbar_init(empty + k, kBW);
        }
        tc::mbar_init(never, 1);
        fence_mbar_init();
        imisc[5] = 0;
    }
    if constexpr (KRES) {
        const char* src = reinterpret_cast<const char*>(Kb + row0 * D);
        char* dst = reinterpret_cast<char*>(smem + L.kres);
        const int pieces = nrows * ROWB / 16;
        for (int c = tid; c < pieces; c += kBT) cp_async16(dst + (size_t)c * 16, src + (size_t)c * 16);
        cp_async_wait_all();
    }
    __syncthreads();
    if (warp == 0) refill();
    {
        if constexpr (KRES) {
            key_rows<T, D, true, KBAR>(kres, 0, nrows, kbr, kbr, dotb, warp, lane);
        } else {
            for (int t = 0; t < NKT; ++t) {
                const T* st = reinterpret_cast<const T*>(acquire());
                key_rows<T, D, true, KBAR>(st, t * KTR, std::min(KTR, nrows - t * KTR), kbr, kbr, dotb, warp, lane);
                release();
            }
        }
    }
    __syncthreads();
    float lmax = -INFINITY;
    for (int row = tid; row < nrows; row += kBT) lmax = fmaxf(lmax, dotb[row]);
    lmax = warp_max(lmax);
    __shared__ float wmax[kBW];
    if (lane == 0) wmax[warp] = lmax;
    __syncthreads();
    if (warp == 0) {
        float v = lane < kBW ? wmax[lane] : -INFINITY;
        v = warp_max(v);
        if (lane == 0) misc[0] = v;
    }
    cluster.sync();
    if (warp == 0) {
        float v = -INFINITY;
        if (lane < G) v = *cluster.map_shared_rank(&misc[0], lane);
        v = warp_max(v);
        if (lane == 0) misc[1] = v;
    }
    __syncthreads();
    const float MK = misc[1];
    const float beta = a.beta;
    for (int row = tid; row < Rpad; row += kBT) dbuf[row] = row < nrows ? expf(beta * (dotb[row] - MK)) : 0.f;
    __syncthreads();
    for (int ch = warp; ch < nch; ch += kBW) {
        const float4 v = reinterpret_cast<const float4*>(dbuf + ch * kChunk)[lane];
        const double incl = warp_scan_incl(quad_sum(v.x, v.y, v.z, v.w), lane);
        if (lane == 31) csl[ch] = incl;
    }
    __syncthreads();
    publish(0, 0);

    // ---------------- r sequential steps ----------------
    float4 flast[kMaxQPT];
#pragma unroll
    for (int k = 0; k < kMaxQPT; ++k) flast[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    int i = 0;
    for (; i < r; ++i) {
        const int cur = i & 1, nxt = cur ^ 1;
        const float* dcur = dbuf + (size_t)cur * Rpad;
        float* dnxt = dbuf + (size_t)nxt * Rpad;
        const double* ib = inbox + (size_t)cur * G * kInbox;

        // -- pivot search (warp 0 of every CTA, identical arithmetic) --
        if (warp == 0) {
            int s = -1;
            const bool any_abort = __any_sync(FULL, lane < G && ib[lane * kInbox + kNchMax + 1] != 0.0);
            if (any_abort) {
                s = -1;
            } else if (a.S_fixed) {
                const int sf = a.S_fixed[b * r + i];
                s = (sf >= 0 && (int64_t)sf < n) ? sf : -1;
            } else {
                const double tcta = lane < G ? ib[lane * kInbox + kNchMax] : 0.0;
                const double incl = warp_scan_incl(tcta, lane);
                const double Tot = __shfl_sync(FULL, incl, 31);
                const unsigned pos_cta = __ballot_sync(FULL, tcta > 0.0);
                if (Tot > 0.0 && pos_cta) {
                    const double t = u_next * Tot;
                    // owner CTA: first with positive mass whose running total reaches t
                    unsigned m = __ballot_sync(FULL, tcta > 0.0 && incl >= t);
                    const int owner = m ? __ffs(m) - 1 : 31 - __clz(pos_cta);
                    const double t1 = t - __shfl_sync(FULL, incl - tcta, owner);
                    // owner's chunk: lane l holds chunks 2l and 2l + 1
                    const double* oc = ib + owner * kInbox;
                    const double c0 = 2 * lane < nch ? oc[2 * lane] : 0.0;
                    const double c1 = 2 * lane + 1 < nch ? oc[2 * lane + 1] : 0.0;
                    const double e = c0 + c1;
                    const double ei = warp_scan_incl(e, lane);
                    const unsigned pos_pair = __ballot_sync(FULL, e > 0.0);
                    m = __ballot_sync(FULL, e > 0.0 && ei >= t1);
                    // a positive total implies a positive chunk; the guard keeps every index in range regardless
                    const int lp = m ? __ffs(m) - 1 : (pos_pair ? 31 - __clz(pos_pair) : 0);
                    if (pos_pair) {  // warp-uniform
                        const double ex = __shfl_sync(FULL, ei - e, lp);
                        const double p0 = __shfl_sync(FULL, c0, lp), p1 = __shfl_sync(FULL, c1, lp);
                        int chunk;
                        double cum;
                        if (p0 > 0.0 && (ex + p0 >= t1 || !(p1 > 0.0))) {
                            chunk = 2 * lp;
                            cum = ex;
                        } else {
                            chunk = 2 * lp + 1;
                            cum = ex + p0;
                        }
                        const double t2 = t1 - cum;
                        // row inside the chunk: one read of the owner's residuals (lane l: rows 4l..4l+3)
                        const float4 v4 =
                            *cluster.map_shared_rank(reinterpret_cast<const float4*>(dcur + chunk * kChunk) + lane, owner);
                        const float vals[4] = {v4.x, v4.y, v4.z, v4.w};
                        const double part = quad_sum(v4.x, v4.y, v4.z, v4.w);
                        double c = warp_scan_incl(part, lane) - part;
                        int hit = -1, lastnz = -1;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float v = vals[k];
                            if (v > 0.f) lastnz = k;
                            c += (double)v;
                            if (hit < 0 && v > 0.f && c >= t2) hit = k;
                        }
                        const unsigned hm = __ballot_sync(FULL, hit >= 0);
                        int local = -1;
                        if (hm) {
                            const int src = __ffs(hm) - 1;
                            local = src * 4 + __shfl_sync(FULL, hit, src);
                        } else {
                            const unsigned nm = __ballot_sync(FULL, lastnz >= 0);
                            if (nm) {
                                const int src = 31 - __clz(nm);
                                local = src * 4 + __shfl_sync(FULL, lastnz, src);
                            }
                        }
                        if (local >= 0) s = (int)((int64_t)owner * R + (int64_t)chunk * kChunk + local);
                    }
                }
            }
            if (lane == 0) {
                imisc[3] = s;
                imisc[4] = 0;
            }
        }
        __syncthreads();
        const int s = imisc[3];
        if (s < 0) break;

        // -- the pivot's factor row (async, needed from the factor pass on) and key --
        for (int j = tid; j < i; j += kBT) cp_async4(fs + j, Fb + (int64_t)j * n + s);
        asm volatile("cp.async.commit_group;" ::: "memory");
        float xr[EPL];
        {
            float4 raw;
            if constexpr (KRES) {
                const int owner = (int)(s / R), lrow = (int)(s - (int64_t)owner * R);
                raw = *cluster.map_shared_rank(
                    reinterpret_cast<const float4*>(kres + (size_t)lrow * D + kl_part * EPL), owner);
            } else {
                raw = __ldg(reinterpret_cast<const float4*>(Kb + (int64_t)s * D + kl_part * EPL));
            }
            widen<T, EPL>(raw, xr);
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                if constexpr (KBAR) xr[e] -= kbr[e];
        }
        if (crank == 0) {
            if (tid == 0 && a.S) a.S[b * r + i] = s;
            if (a.K_S) {
                T* dst = reinterpret_cast<T*>(a.K_S) + (b * r + i) * D;
                for (int c = tid; c < D; c += kBT) dst[c] = Kb[(int64_t)s * D + c];
            }
        }

        // -- key pass: <k_l - kbar, k_s - kbar> for the CTA's rows --
        if constexpr (KRES) {
            key_rows<T, D, false, KBAR>(kres, 0, nrows, xr, kbr, dotb, warp, lane);
        } else {
            for (int t = 0; t < NKT; ++t) {
                const T* st = reinterpret_cast<const T*>(acquire());
                key_rows<T, D, false, KBAR>(st, t * KTR, std::min(KTR, nrows - t * KTR), xr, kbr, dotb, warp, lane);
                release();
            }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();

        // -- pivot residual g_s (warp 0, the same on every CTA) --
        if (warp == 0) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) dot = fmaf(xr[e], xr[e], dot);
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(FULL, dot, o);
            float acc = 0.f;
            for (int j = lane; j < i; j += 32) acc = fmaf(fs[j], fs[j], acc);
            acc = warp_sum(acc);
            if (lane == 0) {
                const float gs = expf(beta * (dot - MK)) - acc;
                misc[2] = gs;
                imisc[4] = !(gs > a.eps);  // max_l h(k_l, k_l) is exp(0) = 1
            }
        }

        // -- factor pass: acc_l = sum_{j < i} F[j, l] F[j, s] --
        float4 acc[kMaxQPT];
#pragma unroll
        for (int k = 0; k < kMaxQPT; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int nft = ntiles(i) - NKT;
        for (int t = 0; t < nft; ++t) {
            const float* st = reinterpret_cast<const float*>(acquire());
            const int c0 = t * CPT, nc = std::min(CPT, i - 1 - c0);
            for (int cc = g; cc < nc; cc += JG) {
                const float f = fs[c0 + cc];
                const float4* col = reinterpret_cast<const float4*>(st + (size_t)cc * R);
#pragma unroll
                for (int k = 0; k < kMaxQPT; ++k) {
                    if (k >= QPT) break;
                    const int q = tt + k * TPG;
                    if (4 * q < nrows) {
                        const float4 v = col[q];
                        acc[k].x = fmaf(v.x, f, acc[k].x);
                        acc[k].y = fmaf(v.y, f, acc[k].y);
                        acc[k].z = fmaf(v.z, f, acc[k].z);
                        acc[k].w = fmaf(v.w, f, acc[k].w);
                    }
                }
            }
            release();
        }
        if (g == 0 && i >= 1) {
            const float f = fs[i - 1];
#pragma unroll
            for (int k = 0; k < kMaxQPT; ++k) {
                acc[k].x = fmaf(flast[k].x, f, acc[k].x);
                acc[k].y = fmaf(flast[k].y, f, acc[k].y);
                acc[k].z = fmaf(flast[k].z, f, acc[k].z);
                acc[k].w = fmaf(flast[k].w, f, acc[k].w);
            }
        }
        if (JG > 1 && g > 0) red[(size_t)(g - 1) * TPG + tt] = acc[0];
        __syncthreads();
        if (imisc[4]) break;

        // -- epilogue (group 0): new column, residual update, chunk sums --
        const float gs = misc[2];
        const float piv = sqrtf(gs);
        if (g == 0) {
            for (int h = 0; h + 1 < JG; ++h) {
                const float4 v = red[(size_t)h * TPG + tt];
                acc[0].x += v.x;
                acc[0].y += v.y;
                acc[0].z += v.z;
                acc[0].w += v.w;
            }
#pragma unroll
            for (int k = 0; k < kMaxQPT; ++k) {
                if (k >= QPT) break;
                const int q = tt + k * TPG, row = 4 * q;
                double p = 0.0;
                if (row < nrows) {
                    const float4 dt = *reinterpret_cast<const float4*>(dotb + row);
                    const float4 dc = *reinterpret_cast<const float4*>(dcur + row);
                    const float dts[4] = {dt.x, dt.y, dt.z, dt.w}, dcs[4] = {dc.x, dc.y, dc.z, dc.w};
                    const float as[4] = {acc[k].x, acc[k].y, acc[k].z, acc[k].w};
                    float fo[4], dn[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int64_t l = row0 + row + e;
                        float gl = expf(beta * (dts[e] - MK)) - as[e];
                        if (l == s) gl = gs;
                        fo[e] = gl / piv;
                        dn[e] = fmaxf(dcs[e] - fo[e] * fo[e], 0.f);
                        if (l == s) dn[e] = 0.f;
                    }
                    flast[k] = make_float4(fo[0], fo[1], fo[2], fo[3]);
                    *reinterpret_cast<float4*>(Fb + (int64_t)i * n + row0 + row) = flast[k];
                    *reinterpret_cast<float4*>(dnxt + row) = make_float4(dn[0], dn[1], dn[2], dn[3]);
                    p = quad_sum(dn[0], dn[1], dn[2], dn[3]);
                } else if (row < Rpad) {
                    *reinterpret_cast<float4*>(dnxt + row) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                const double incl = warp_scan_incl(p, lane);
                const int ch = (tt >> 5) + k * (TPG >> 5);
                if (lane == 31 && ch < nch) csl[ch] = incl;
            }
            fence_async_global();  // the column is read by bulk copies two steps on
        }
        __syncthreads();
        done_step = i + 1;
        publish(nxt, i + 1);
    }

    // ---------------- drain the ring, effective rank, padding past it ----------------
    if (tid == 0) {
        const unsigned long long lim = imisc[5] ? 10000000ull : kWaitLimitNs;
        int slot = c_slot;
        unsigned par = c_par;
        for (long long t = tcons; t < tiss; ++t) {
            if (!tc::mbar_wait(full + slot, par, lim)) {
                set_abort();
                break;
            }
            if (++slot == NS) {
                slot = 0;
                par ^= 1u;
            }
        }
    }
    const int rr = i;
    for (int j = rr; j < r; ++j) {
        float* dst = Fb + (int64_t)j * n + row0;
        for (int row = tid; row < nrows; row += kBT) dst[row] = 0.f;
    }
    if (crank == 0) {
        if (tid == 0) a.rank[b] = rr;
        for (int j = rr + tid; j < r; j += kBT)
            if (a.S) a.S[b * r + j] = -1;
        if (a.K_S) {
            T* dst = reinterpret_cast<T*>(a.K_S) + b * r * D;
            for (int64_t e = (int64_t)rr * D + tid; e < (int64_t)r * D; e += kBT) dst[e] = T(0.f);
        }
    }
    __syncthreads();
    // keep this CTA's shared memory alive until every peer is done reading it
    cluster.sync();
}

template <typename E, int D, bool KRES, bool KBAR>
cudaError_t launch_t(const BulkArgs& a, size_t smem, cudaStream_t stream, int* max_clusters) {
    auto kern = rpc_select_bulk_kernel<E, D, KRES, KBAR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.G > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(max_clusters ? a.G : a.BH * a.G));
    cfg.blockDim = dim3(kBT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_clusters) {
        *max_clusters = 0;
        e = cudaOccupancyMaxActiveClusters(max_clusters, kern, &cfg);
        if (e != cudaSuccess) cudaGetLastError();
        return e;
    }
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename E, int D>
cudaError_t dispatch_flags(bool kres, bool kbar, const BulkArgs& a, size_t smem, cudaStream_t st, int* mc) {
    if (kres) return kbar ? launch_t<E, D, true, true>(a, smem, st, mc) : launch_t<E, D, true, false>(a, smem, st, mc);
    return kbar ? launch_t<E, D, false, true>(a, smem, st, mc) : launch_t<E, D, false, false>(a, smem, st, mc);
}

cudaError_t dispatch(int dtype, int d, bool kres, bool kbar, const BulkArgs& a, size_t smem, cudaStream_t st,
                     int* mc) {
    if (dtype == 1) {
        switch (d) {
            case 32: return dispatch_flags<BF16, 32>(kres, kbar, a, smem, st, mc);
            case 64: return dispatch_flags<BF16, 64>(kres, kbar, a, smem, st, mc);
            case 128: return dispatch_flags<BF16, 128>(kres, kbar, a, smem, st, mc);
        }
    } else {
        switch (d) {
            case 32: return dispatch_flags<F32, 32>(kres, kbar, a, smem, st, mc);
            case 64: return dispatch_flags<F32, 64>(kres, kbar, a, smem, st, mc);
            case 128: return dispatch_flags<F32, 128>(kres, kbar, a, smem, st, mc);
        }
    }
    return cudaErrorInvalidValue;
}

// Shape of the kernel for n keys over G CTAs; false when it does not apply.
bool plan_bulk(int64_t n, int r, int d, int dtype, int G, BulkArgs* a, size_t* smem, bool* kres) {
    if (n % 4 != 0) return false;
    const int R = (int)round_up(ceil_div(n, G), 4);
    if (R > kNchMax * kChunk) return false;
    const int bK = dtype == 1 ? 2 : 4;
    const int rowb = d * bK;
    const int Q = R / 4;
    int TPG, JG, QPT;
    if (Q >= kBT) {
        TPG = kBT;
        JG = 1;
        QPT = (int)ceil_div(Q, kBT);
    } else {
        TPG = 32;
        while (TPG < Q) TPG *= 2;
        JG = kBT / TPG;
        QPT = 1;
    }
    if (QPT > kMaxQPT) return false;
    a->G = G;
    a->R = R;
    a->CPT = kStageBytes / (4 * R);
    a->KTR = kStageBytes / rowb;
    a->NKT = (int)ceil_div(R, a->KTR);
    a->JG = JG;
    a->TPG = TPG;
    a->QPT = QPT;
    auto bytes = [&](int ns, bool kr) { return BulkLayout(R, r, rowb, ns, G, JG, TPG, kr).total; };
    // resident keys when at least two stages remain; otherwise stream them
    for (const bool kr : {true, false}) {
        int ns = 0;
        while (ns + 1 <= kMaxStages && bytes(ns + 1, kr) <= kSmemCap) ++ns;
        if (ns >= (kr ? 2 : 3)) {
            a->NS = ns;
            *kres = kr;
            *smem = bytes(ns, kr);
            return true;
        }
    }
    return false;
}

}  // namespace

void set_select_force_timeout(unsigned long long ns) { g_force_select_timeout_ns = ns; }
unsigned long long select_force_timeout_ns() { return g_force_select_timeout_ns; }

int read_select_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_select_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_select_status, &z, sizeof(int));
    }
    return v;
}

// Launch the bulk-copy kernel; G_override > 0 fixes the cluster size, else
// the shared chooser picks it from the occupancy of this kernel's shapes.
// *used = false when the shape is not one this kernel handles (the caller
// then takes the cp.async kernel).
Status launch_select_bulk(const SelectRequest& q, int G_override, cudaStream_t stream, bool* used, int* G_used) {
    *used = false;
    if (reinterpret_cast<uintptr_t>(q.K) % 16 != 0 || reinterpret_cast<uintptr_t>(q.F) % 16 != 0) return Status::ok();
    if (q.d != 32 && q.d != 64 && q.d != 128) return Status::ok();
    BulkArgs a{};
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
    a.force_timeout_ns = g_force_select_timeout_ns;
    int G = G_override;
    if (G <= 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        const ClusterKey key{dev, 2, q.n, q.BH, q.r, q.d, q.dtype};
        G = cached_cluster_lookup(key);
        if (G <= 0) {
            struct Ctx {
                const SelectRequest* q;
                cudaStream_t stream;
            } ctx{&q, stream};
            G = choose_cluster_rows(q.n, q.BH, [](int g, void* p) -> int {
                const Ctx& c = *static_cast<const Ctx*>(p);
                BulkArgs t{};
                size_t sm = 0;
                bool kr = false;
                if (!plan_bulk(c.q->n, c.q->r, c.q->d, c.q->dtype, g, &t, &sm, &kr)) return 0;
                t.G = g;
                int mc = 0;
                if (dispatch(c.q->dtype, c.q->d, kr, c.q->kbar != nullptr, t, sm, c.stream, &mc) != cudaSuccess) return 0;
                return mc;
            }, &ctx, nullptr);
            if (G <= 0) return Status::ok();
            cached_cluster_store(key, G);
        }
    }
    size_t smem = 0;
    bool kres = false;
    if (!plan_bulk(q.n, q.r, q.d, q.dtype, G, &a, &smem, &kres)) return Status::ok();
    *used = true;
    *G_used = G;
    cudaError_t err = dispatch(q.dtype, q.d, kres, q.kbar != nullptr, a, smem, stream, nullptr);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return Status::cuda(err, "select (bulk) launch");
    return Status::ok();
}

}  // namespace wildcat
