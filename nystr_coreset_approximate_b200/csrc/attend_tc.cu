// attend_tc.cu -- weighted-coreset attention on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2 plug-in
// estimator and Alg. 3 WtdAttn, for bfloat16 inputs:
//     P = exp(beta Q K_S^T - beta m),  N = P V_S,  D = P w,  O = clip(N / D)
// with a shift m_i = |q_i| max_l |k_S,l| per query row: every exponent is
// <= 0, and the shift cancels in N / D like any per-row constant (the
// CUDA-core kernel and the oracle use one shift per instance; the ratio is
// the same).  The row's shift comes from the query tile already in shared
// memory, so no separate pass over Q is needed.
//
// Persistent CTAs (one per SM, 16 warps) walk units of two 128-query tiles
// of one instance; each unit walks the coreset in chunks of 128 rows.  Warp
// roles (setmaxnreg gives the softmax and epilogue groups the registers):
//   warp 0     producer (one thread): TMA loads of each unit's two Q tiles
//              (a slot's next tile as soon as its last GEMM1 and its row norms
//              are done), of each K_S chunk and of each V_S^T chunk plus its
//              slice of w, into 128-byte-swizzled shared memory, NS stages
//   warp 1     tensor cores (one thread issues):
//                GEMM1  S_t = Q_t K_S,c^T   tcgen05.mma kind::f16, M = 128,
//                       N = 128, both operands in shared memory, fp32 in TMEM
//                GEMM2  O_t += P_t V_S,c    A operand P_t read from TMEM
//                       (where the softmax threads left it), N = d
//              as one stream per tile slot, G2(c, t) then G1(c + 1, t), the two
//              slots alternating: while one slot's scores are exponentiated
//              the other slot's products run, and a slot's next unit follows
//              its last chunk without a break
//   warps 2-3  idle (they keep the four groups below one warp per SM
//              sub-partition each)
//   warps 4-7  softmax of slot 0, warps 8-11 of slot 1: thread i of the group
//              owns query row i (= TMEM lane i).  Per unit it forms its row's
//              shift from the Q tile in shared memory; per chunk it reads its
//              128 scores with tcgen05.ld (the next 32 columns in flight while
//              it works on these), forms P = 2^(s beta log2e - m_i beta log2e)
//              on the special-function unit, rounds P once to bf16, writes the
//              packed pairs back over the scores (tcgen05.st) for GEMM2 and
//              accumulates D = sum_l P_l w_l in fp32 (packed fp32x2 FMAs); at
//              the unit's end it leaves D in shared memory
//   warps 12-15 epilogue: per tile it reads the rows of O from TMEM (half the
//              columns at a time, releasing the accumulator after the second
//              half), forms clip(N / D, v_min, v_max), stages 128 x 32 boxes
//              in two shared-memory buffers and stores them with TMA
// The tensor pipe bounds the kernel: on this part one 128 x 128 x 16 MMA
// takes about 124 cycles with both operands in shared memory and 136 with
// A in tensor memory (a probe of back-to-back MMAs: 4.2 and 3.9 kflop per
// clock per SM, against about 6.2 for a 128 x 256 x 16 MMA), so a unit's 16
// products need about 16.6k cycles, and a unit takes about 20k.
// Tensor memory (512 columns): O_0, O_1 (d columns each), S_0, S_1 (128 each).
// V_S and w are prepared per call: V_S^T rounded to bf16 (its bf16 rounding
// leaves the plug-in estimator within 6.1e-4 of the value range on every
// workload here, against a bound of 2e-2) and w zero-padded, both zero past
// the instance's rank.  Keys at or past the rank get P = 0.
//
// Every mbarrier wait is bounded (2 s) and gives up when another role has
// given up; an expired wait records WILDCAT_ERR_TIMEOUT in the device status
// word, the CTA drains the copies and tensor-core work it issued (bounded),
// frees its tensor memory and returns.  No load uses cluster multicast.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace wildcat {

__device__ int g_device_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        else
            cudaGetLastError();
    });
    if (!encode || (reinterpret_cast<uintptr_t>(base) & 15u) || (s1 & 15u) || (s2 & 15u) ||
        b0 * (uint32_t)elem_bytes != 128u)
        return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return encode(map, type, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using namespace tc;

constexpr int kRows = 128;    // queries per tile = TMEM lanes
constexpr int kChunk = 128;   // coreset rows per chunk = N of GEMM1
constexpr int kWarps = 16;    // producer / tensor cores, two softmax groups, one epilogue group
constexpr int kThreads = kWarps * 32;
// registers per thread after the split (launched with 65536 / 512 = 128 each):
// warps 0-3 (producer, tensor cores, two idle) give up some to the softmax
// and epilogue groups; per sub-partition 88 + 2 * 144 + 136 = 512 = 16384 / 32.
constexpr int kRegsLow = 88, kRegsSoftmax = 144, kRegsEpilogue = 136;
static_assert(kRegsLow + 2 * kRegsSoftmax + kRegsEpilogue == 512, "register split");
constexpr unsigned long long kDrainNs = 100000000ull;  // 100 ms for work in flight after an abort
unsigned long long g_force_timeout_ns = 0;             // test hook, 0 = off

template <int NS>
struct Bars {
    uint64_t q_full[2], q_free[2];
    uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2], den_full[2];
    uint64_t drain, never;
    unsigned tmem_base;
    int abort;
};

template <int D>
struct Cfg {
    static constexpr int NS = D == 128 ? 2 : 4;          // stages per operand ring
    static constexpr int KB = D / 64;                    // 128-byte blocks per Q / K_S row
    static constexpr uint32_t q_bytes = kRows * D * 2;   // one Q tile
    static constexpr uint32_t k_bytes = kChunk * D * 2;  // one K_S chunk
    static constexpr uint32_t v_bytes = D * kChunk * 2;  // one V_S^T chunk
    static constexpr uint32_t w_bytes = kChunk * 4;      // one chunk of w
    static constexpr uint32_t o_bytes = kRows * 128;     // one output box: 128 rows x 32 fp32
    static constexpr uint32_t off_q = 0;
    static constexpr uint32_t off_k = off_q + 2 * q_bytes;
    static constexpr uint32_t off_v = off_k + NS * k_bytes;
    static constexpr uint32_t off_o = off_v + NS * v_bytes;  // the epilogue group's two output boxes
    static constexpr uint32_t off_w = off_o + 2 * o_bytes;
    static constexpr uint32_t off_den = off_w + NS * w_bytes;  // row denominators, [2][128]
    static constexpr uint32_t off_bar = off_den + 2 * kRows * 4;
    static constexpr uint32_t total = off_bar + (uint32_t)sizeof(Bars<NS>);
    static constexpr unsigned tmem_cols = 512;
    static constexpr unsigned col_O = 0;       // O_t at col_O + t * D
    static constexpr unsigned col_S = 2 * D;   // S_t at col_S + t * kChunk
    static_assert(2 * D + 2 * kChunk <= 512, "tensor memory");
    static_assert(total <= 232448, "shared memory");
};

// The work of one CTA is a sequence of units (two query tiles of one
// instance): unit u covers queries [256 j, 256 j + 256) of instance u / upi,
// j = u % upi.  Every role walks the same sequence.  A second tile that lies
// past m loads zeros and has its stores dropped by the tensor map bounds, so
// every unit has the same two-tile shape.
struct Unit {
    int b, nch;
    int64_t i0;
};
__device__ __forceinline__ Unit unit_at(int64_t u, int64_t upi, int64_t m, const int32_t* rank) {
    // the host keeps the unit count below 2^31, so 32-bit division suffices
    Unit w;
    const uint32_t uu = (uint32_t)u, up = (uint32_t)upi;
    w.b = (int)(uu / up);
    w.i0 = (int64_t)(uu - (uint32_t)w.b * up) * (2 * kRows);
    w.nch = (rank[w.b] + kChunk - 1) / kChunk;
    return w;
}

// State shared by the roles of one CTA.
template <int D>
struct Ctx {
    unsigned char* sm;
    unsigned sbase, tmem;
    Bars<Cfg<D>::NS>* bars;
    volatile int* abort_flag;
    int64_t m, upi, units;
    const int32_t* rank;
    __device__ void give_up() const {
        *abort_flag = 1;
        atomicExch(&g_device_status, 5);
    }
};

template <int D>
__device__ __forceinline__ void role_producer(const Ctx<D>& x, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                              const CUtensorMap* tmV, const float* __restrict__ wpad, int rpad) {
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    auto* bars = x.bars;
    prefetch_tmap(tmQ);
    prefetch_tmap(tmK);
    prefetch_tmap(tmV);
    int64_t g = 0;       // chunks issued over this CTA's units
    int qn0 = 0, qn1 = 0;  // Q tiles loaded into slot 0 / 1
    bool ok = true;
    for (int64_t u = blockIdx.x; u < x.units && ok; u += gridDim.x) {
        const Unit w = unit_at(u, x.upi, x.m, x.rank);
        if (w.nch == 0) continue;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            int& qn = t ? qn1 : qn0;
            // the slot's previous tile: its last GEMM1 done and its row norms read
            if (qn > 0 && !(ok = mbar_wait_suspend(&bars->q_free[t], (unsigned)(qn - 1) & 1u, x.abort_flag))) break;
            mbar_expect_tx(&bars->q_full[t], C::q_bytes);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(x.sbase + C::off_q + t * C::q_bytes + kb * (kRows * 128), tmQ, kb * 64,
                            (int)(w.i0 + t * kRows), w.b, &bars->q_full[t]);
            ++qn;
        }
        for (int c = 0; c < w.nch && ok; ++c, ++g) {
            const int s = (int)(g % NS);
            const unsigned ph = (unsigned)(g / NS) & 1u;
            if (g >= NS && !(ok = mbar_wait_suspend(&bars->k_empty[s], ph ^ 1u, x.abort_flag))) break;
            mbar_expect_tx(&bars->k_full[s], C::k_bytes);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(x.sbase + C::off_k + s * C::k_bytes + kb * (kChunk * 128), tmK, kb * 64, c * kChunk, w.b,
                            &bars->k_full[s]);
            if (g >= NS && !(ok = mbar_wait_suspend(&bars->v_empty[s], ph ^ 1u, x.abort_flag))) {
                ++g;  // this chunk's K copy is in flight
                break;
            }
            mbar_expect_tx(&bars->v_full[s], C::v_bytes + C::w_bytes);
#pragma unroll
            for (int j = 0; j < kChunk / 64; ++j)
                tma_load_3d(x.sbase + C::off_v + s * C::v_bytes + j * (D * 128), tmV, c * kChunk + j * 64, 0, w.b,
                            &bars->v_full[s]);
            bulk_load(x.sbase + C::off_w + s * C::w_bytes, wpad + (int64_t)w.b * rpad + (int64_t)c * kChunk,
                      C::w_bytes, &bars->v_full[s]);
        }
    }
    if (!ok) x.give_up();
    if (*x.abort_flag) {
        // copies still in flight land before the CTA's shared memory is released
        if (qn0 > 0) mbar_wait(&bars->q_full[0], (unsigned)(qn0 - 1) & 1u, kDrainNs);
        if (qn1 > 0) mbar_wait(&bars->q_full[1], (unsigned)(qn1 - 1) & 1u, kDrainNs);
        for (int64_t c = g > NS ? g - NS : 0; c < g; ++c) {
            mbar_wait(&bars->k_full[c % NS], (unsigned)(c / NS) & 1u, kDrainNs);
            mbar_wait(&bars->v_full[c % NS], (unsigned)(c / NS) & 1u, kDrainNs);
        }
    }
}

template <int D>
__device__ __forceinline__ void gemm1(const Ctx<D>& x, int64_t g, int t) {  // S_t = Q_t K_g^T
    using C = Cfg<D>;
    const unsigned qa = x.sbase + C::off_q + t * C::q_bytes;
    const unsigned kb = x.sbase + C::off_k + (unsigned)(g % C::NS) * C::k_bytes;
    const uint64_t da = umma_desc(qa), db = umma_desc(kb);
    const uint32_t hi = (uint32_t)(da >> 32);  // the same for both operands (layout and swizzle fields)
    const uint32_t a_lo = (uint32_t)da, b_lo = (uint32_t)db;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        // descriptor start addresses advance in 16-byte units
        const uint32_t oa = (uint32_t)(((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4);
        const uint32_t ob = (uint32_t)(((kk >> 2) * (kChunk * 128) + (kk & 3) * 32) >> 4);
        mma_bf16_w(x.tmem + C::col_S + t * kChunk, a_lo + oa, hi, b_lo + ob, hi, idesc_bf16(128, kChunk), kk > 0);
    }
}
template <int D>
__device__ __forceinline__ void gemm2(const Ctx<D>& x, int64_t g, int t, bool first) {  // O_t (+)= P_t V_g
    using C = Cfg<D>;
    const unsigned vb = x.sbase + C::off_v + (unsigned)(g % C::NS) * C::v_bytes;
    const uint64_t db = umma_desc(vb);
    const uint32_t hi = (uint32_t)(db >> 32), b_lo = (uint32_t)db;
#pragma unroll
    for (int kk = 0; kk < kChunk / 16; ++kk) {
        const uint32_t ob = (uint32_t)(((kk >> 2) * (D * 128) + (kk & 3) * 32) >> 4);
        mma_bf16_ts_w(x.tmem + C::col_O + t * D, x.tmem + C::col_S + t * kChunk + kk * 8, b_lo + ob, hi,
                      idesc_bf16(128, D), (!first || kk > 0) ? 1 : 0);
    }
}

// Position in the CTA's stream of chunks: unit u, its chunk c of nch, the
// global chunk index g (over all of this CTA's units).
struct Step {
    int64_t u, g;
    int c, nch;
    Unit w;
};
// The chunk after `s`, skipping units of rank 0; false at the end.
__device__ __forceinline__ bool next_step(Step& s, int64_t units, int64_t upi, int64_t m, const int32_t* rank) {
    if (s.c + 1 < s.nch) {
        ++s.c;
        ++s.g;
        return true;
    }
    for (int64_t u = s.u + gridDim.x; u < units; u += gridDim.x) {
        const Unit w = unit_at(u, upi, m, rank);
        if (w.nch == 0) continue;
        s.u = u;
        s.w = w;
        s.c = 0;
        s.nch = w.nch;
        ++s.g;
        return true;
    }
    return false;
}

// GEMM2 of chunk `cur` for tile slot T, then GEMM1 of the slot's next chunk
// (the next unit's first chunk after a unit's last): each slot runs one
// continuous stream, so the stagger between the two slots (one exponentiates
// while the other's products run) carries over unit boundaries.  Returns
// false when a wait gave up.
template <int D, int T>
__device__ __forceinline__ bool mma_slot_step(const Ctx<D>& x, const Step& cur, const Step& nxt, bool has_next,
                                              int& ct, int& on, int& qn) {
    using C = Cfg<D>;
    auto* bars = x.bars;
    if (!mbar_wait_suspend(&bars->p_full[T], (unsigned)ct & 1u, x.abort_flag)) return false;
    ct ^= 1;
    // the epilogue group has taken the slot's previous O out of tensor memory
    if (cur.c == 0 && on > 0 && !mbar_wait_suspend(&bars->o_free[T], (unsigned)(on - 1) & 1u, x.abort_flag))
        return false;
    tc_fence_after();
    gemm2<D>(x, cur.g, T, cur.c == 0);
    if (cur.c + 1 == cur.nch) {
        mma_commit(&bars->o_full[T]);
        ++on;
    }
    if (has_next) {
        if (T == 0 && !mbar_wait_suspend(&bars->k_full[nxt.g % C::NS], (unsigned)(nxt.g / C::NS) & 1u, x.abort_flag))
            return false;
        if (nxt.c == 0) {  // a new unit: its Q tile for this slot
            if (!mbar_wait_suspend(&bars->q_full[T], (unsigned)qn & 1u, x.abort_flag)) return false;
            qn ^= 1;
        }
        tc_fence_after();
        // issued after GEMM2 of the same slot, which has read P_t out of these
        // columns by the time this product writes them (tcgen05.mma executes in
        // issue order)
        gemm1<D>(x, nxt.g, T);
        mma_commit(&bars->s_full[T]);
        if (nxt.c + 1 == nxt.nch) mma_commit(&bars->q_free[T]);  // the slot's last GEMM1 of that unit
    }
    return true;
}

template <int D>
__device__ __forceinline__ void role_mma(const Ctx<D>& x) {
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    auto* bars = x.bars;
    int qn0 = 0, qn1 = 0;  // Q tiles consumed per slot (parity)
    int ct0 = 0, ct1 = 0;  // chunks of each slot handed to the softmax (parity)
    int on0 = 0, on1 = 0;  // accumulations of each slot's O
    Step cur;
    cur.u = (int64_t)blockIdx.x - gridDim.x;
    cur.c = 0;
    cur.nch = 0;
    cur.g = -1;
    bool ok = true;
    if (next_step(cur, x.units, x.upi, x.m, x.rank)) {
        // the first chunk's GEMM1 for both slots
        ok = mbar_wait_suspend(&bars->k_full[0], 0, x.abort_flag) &&
             mbar_wait_suspend(&bars->q_full[0], 0, x.abort_flag) &&
             mbar_wait_suspend(&bars->q_full[1], 0, x.abort_flag);
        if (ok) {
            qn0 = qn1 = 1;
            tc_fence_after();
            gemm1<D>(x, 0, 0);
            mma_commit(&bars->s_full[0]);
            gemm1<D>(x, 0, 1);
            mma_commit(&bars->s_full[1]);
            if (cur.nch == 1) {
                mma_commit(&bars->q_free[0]);
                mma_commit(&bars->q_free[1]);
            }
            mma_commit(&bars->k_empty[0]);
        }
        while (ok) {
            Step nxt = cur;
            const bool has_next = next_step(nxt, x.units, x.upi, x.m, x.rank);
            if (!(ok = mbar_wait_suspend(&bars->v_full[cur.g % NS], (unsigned)(cur.g / NS) & 1u, x.abort_flag)))
                break;
            ok = mma_slot_step<D, 0>(x, cur, nxt, has_next, ct0, on0, qn0) &&
                 mma_slot_step<D, 1>(x, cur, nxt, has_next, ct1, on1, qn1);
            if (!ok) break;
            mma_commit(&bars->v_empty[cur.g % NS]);
            if (!has_next) break;
            mma_commit(&bars->k_empty[nxt.g % NS]);
            cur = nxt;
        }
    }
    if (!ok) x.give_up();
    // every product issued has finished before tensor memory is released
    mma_commit(&bars->drain);
    mbar_wait(&bars->drain, 0, kDrainNs);
}

// Softmax group t (warps 4 + 4t .. 7 + 4t): thread `row` owns query row `row`
// of tile slot t (TMEM lane `row`).
template <int D>
__device__ __forceinline__ void role_softmax(const Ctx<D>& x, int t, int quad, int lane, float beta,
                                             const float* __restrict__ kmax) {
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    auto* bars = x.bars;
    const int row = quad * 32 + lane;
    const unsigned tS = x.tmem + C::col_S + t * kChunk + ((unsigned)(quad * 32) << 16);
    const float a = beta * 1.4426950408889634f;
    const unsigned char* qrow = x.sm + C::off_q + t * C::q_bytes + row * 128;
    float* den_s = reinterpret_cast<float*>(x.sm + C::off_den);
    int64_t g = 0;
    int qn = 0, ct = 0, on = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < x.units && ok; u += gridDim.x) {
        const Unit w = unit_at(u, x.upi, x.m, x.rank);
        if (w.nch == 0) {
            g += w.nch;
            continue;
        }
        const int rr = x.rank[w.b];
        // per-row shift m_i = |q_i| * max_l |k_S,l| (>= <q_i, k_l>; it cancels in N / D)
        ok = __all_sync(0xffffffffu, mbar_wait_suspend(&bars->q_full[t], (unsigned)qn & 1u, x.abort_flag));
        if (!ok) break;
        float qq = 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 8; ++cc) {
            const uint4 q4 =
                *reinterpret_cast<const uint4*>(qrow + (cc >> 3) * (kRows * 128) + (((cc & 7) ^ (row & 7)) << 4));
            const uint32_t xs[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(xs[e] << 16), hi = __uint_as_float(xs[e] & 0xffff0000u);
                qq = fmaf(lo, lo, qq);
                qq = fmaf(hi, hi, qq);
            }
        }
        const float sh = a * sqrtf(qq) * kmax[w.b];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_free[t]);
        qn ^= 1;
        const float2 a2 = make_float2(a, a), nsh2 = make_float2(-sh, -sh);
        float2 dacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        for (int c = 0; c < w.nch && ok; ++c, ++g) {
            const int s = (int)(g % NS);
            const bool got = mbar_wait_suspend(&bars->s_full[t], (unsigned)ct & 1u, x.abort_flag) &&
                             mbar_wait_suspend(&bars->v_full[s], (unsigned)(g / NS) & 1u, x.abort_flag);
            ok = __all_sync(0xffffffffu, got);  // tcgen05.ld / st below are warp-collective
            if (!ok) break;
            ct ^= 1;
            tc_fence_after();
            const float4* w4 = reinterpret_cast<const float4*>(x.sm + C::off_w + s * C::w_bytes);
            const int lim = rr - c * kChunk;  // keys of this chunk below the rank
            uint32_t v[2][32];
            tmem_ld32_nowait(tS, v[0]);
#pragma unroll
            for (int j = 0; j < kChunk / 32; ++j) {
                tmem_wait_ld();
                if (j + 1 < kChunk / 32) tmem_ld32_nowait(tS + 32 * (j + 1), v[(j + 1) & 1]);
                uint32_t pk[16];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) {
                    const float4 ww = w4[8 * j + e2];
                    float p[4];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int e = 2 * e2 + h;
                        const float2 x2 = ffma2(
                            make_float2(__uint_as_float(v[j & 1][2 * e]), __uint_as_float(v[j & 1][2 * e + 1])), a2,
                            nsh2);
                        p[2 * h] = ex2_approx(x2.x);
                        p[2 * h + 1] = ex2_approx(x2.y);
                    }
                    if (lim < kChunk) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) p[q] = 32 * j + 4 * e2 + q < lim ? p[q] : 0.f;
                    }
                    pk[2 * e2] = pack_bf16x2(p[0], p[1]);
                    pk[2 * e2 + 1] = pack_bf16x2(p[2], p[3]);
                    // denominator in fp32 from the unrounded P (its bf16 rounding in N is
                    // unbiased, 2^-9 relative, far inside the 2e-2 bound)
                    dacc[0] = ffma2(make_float2(p[0], p[1]), make_float2(ww.x, ww.y), dacc[0]);
                    dacc[1] = ffma2(make_float2(p[2], p[3]), make_float2(ww.z, ww.w), dacc[1]);
                }
                tmem_st16(tS + 16 * j, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[t]);
        }
        if (!ok) break;
        // the row's denominator for the epilogue group, once the epilogue has read
        // the slot's previous one (with one chunk per unit this group can finish a
        // unit before the epilogue has taken the previous unit's results)
        if (on > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait_suspend(&bars->o_free[t], (unsigned)(on - 1) & 1u, x.abort_flag));
            if (!ok) break;
        }
        ++on;
        den_s[t * kRows + row] = (dacc[0].x + dacc[0].y) + (dacc[1].x + dacc[1].y);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->den_full[t]);
    }
    if (!ok && lane == 0) x.give_up();
}

// A read-only 16-byte load kept in program order (volatile), so the compiler
// does not hoist a whole row's worth of bounds into registers.
__device__ __forceinline__ float4 ld_nc_f4(const float* p) {
    float4 r;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}

// AND of `v` over the 128 threads of the epilogue group (a group barrier).
__device__ __forceinline__ bool group_all(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}

// One 128 x 32 box of outputs O = clip(v * rcp, lo, hi) from 32 accumulator
// values per thread, through box `buf` of the epilogue group's two
// shared-memory boxes to TMA (the store of the other box may still be reading).
template <int D>
__device__ __forceinline__ void put_box(const Ctx<D>& x, int row, const uint32_t (&v)[32], int col0, float rcp,
                                        const float* lo, const float* hi, int64_t y, int b, const CUtensorMap* tmO,
                                        int buf) {
    using C = Cfg<D>;
    unsigned char* brow = x.sm + C::off_o + buf * C::o_bytes + row * 128;
    if (row == 0) bulk_wait_read_1();  // this box's previous store has read it
    named_barrier_sync(3, 128);
    const float* lb = lo + col0;
    const float* hb = hi + col0;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const float4 l4 = ld_nc_f4(lb + 4 * cc);
        const float4 h4 = ld_nc_f4(hb + 4 * cc);
        float4 o;
        o.x = fminf(fmaxf(__uint_as_float(v[4 * cc + 0]) * rcp, l4.x), h4.x);
        o.y = fminf(fmaxf(__uint_as_float(v[4 * cc + 1]) * rcp, l4.y), h4.y);
        o.z = fminf(fmaxf(__uint_as_float(v[4 * cc + 2]) * rcp, l4.z), h4.z);
        o.w = fminf(fmaxf(__uint_as_float(v[4 * cc + 3]) * rcp, l4.w), h4.w);
        // volatile like the loads above, so each 16-byte group of bounds is consumed
        // before the next is fetched (few registers in flight)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(brow + ((cc ^ (row & 7)) << 4))),
                     "f"(o.x), "f"(o.y), "f"(o.z), "f"(o.w)
                     : "memory");
    }
    fence_async_smem();
    named_barrier_sync(3, 128);
    if (row == 0) {
        tma_store_3d(tmO, col0, (int)y, b, x.sbase + C::off_o + buf * C::o_bytes);
        bulk_commit();
    }
}

// The epilogue of tile slot T of one unit.  Returns false when a wait gave up.
template <int D, int T>
__device__ __forceinline__ bool epilogue_tile(const Ctx<D>& x, const Unit& w, int quad, int lane, int& on,
                                              const CUtensorMap* tmO, const float* lo, const float* hi) {
    using C = Cfg<D>;
    const int row = quad * 32 + lane;
    const int64_t y = w.i0 + T * kRows;
    uint32_t v[D / 64][32];
    if (w.nch == 0) {  // rank 0: 0 / 0 is NaN, which the clip turns into v_min
#pragma unroll
        for (int e = 0; e < 32; ++e) v[0][e] = 0u;
#pragma unroll 1
        for (int col0 = 0; col0 < D; col0 += 32)
            put_box<D>(x, row, v[0], col0, __int_as_float(0x7f800000), lo, hi, y, w.b, tmO, (col0 >> 5) & 1);
        return true;
    }
    const bool got = mbar_wait_suspend(&x.bars->o_full[T], (unsigned)on & 1u, x.abort_flag) &&
                     mbar_wait_suspend(&x.bars->den_full[T], (unsigned)on & 1u, x.abort_flag);
    // all four warps agree before the group barriers of put_box
    if (!group_all(3, got)) return false;
    ++on;
    tc_fence_after();
    const unsigned tO = x.tmem + C::col_O + T * D + ((unsigned)(quad * 32) << 16);
    const float rcp = 1.0f / reinterpret_cast<const float*>(x.sm + C::off_den)[T * kRows + row];
    constexpr int H = D / 2;  // columns per half
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < H / 32; ++k) tmem_ld32_nowait(tO + h * H + 32 * k, v[k]);
        tmem_wait_ld();
        if (h == 1) {
            // the slot's accumulator and denominator are read: release them (the
            // slot's next GEMM2 comes after the next chunk's softmax, well later)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&x.bars->o_free[T]);
        }
#pragma unroll
        for (int k = 0; k < H / 32; ++k)
            put_box<D>(x, row, v[k], h * H + 32 * k, rcp, lo, hi, y, w.b, tmO, (h * (H / 32) + k) & 1);
    }
    return true;
}

// Epilogue group (warps 12-15): O = clip(N / D) for every tile, in unit order.
template <int D>
__device__ __forceinline__ void role_epilogue(const Ctx<D>& x, int quad, int lane, const CUtensorMap* tmO,
                                              const float* __restrict__ vmin, const float* __restrict__ vmax) {
    int on0 = 0, on1 = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < x.units && ok; u += gridDim.x) {
        const Unit w = unit_at(u, x.upi, x.m, x.rank);
        const float* lo = vmin + (int64_t)w.b * D;
        const float* hi = vmax + (int64_t)w.b * D;
        ok = epilogue_tile<D, 0>(x, w, quad, lane, on0, tmO, lo, hi) &&
             epilogue_tile<D, 1>(x, w, quad, lane, on1, tmO, lo, hi);
    }
    if (!ok && lane == 0) x.give_up();
    if (quad == 0 && lane == 0) bulk_wait_all();
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const float* __restrict__ wpad, int rpad, int64_t m, int64_t BH,
                     const int32_t* __restrict__ rank, float beta, const float* __restrict__ vmin,
                     const float* __restrict__ vmax, const float* __restrict__ kmax,
                     unsigned long long force_timeout_ns) {
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ __align__(1024) unsigned char sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    Ctx<D> x;
    x.sm = sm;
    x.sbase = smem_u32(sm);
    x.bars = reinterpret_cast<Bars<NS>*>(sm + C::off_bar);
    x.abort_flag = &x.bars->abort;
    x.m = m;
    x.upi = (m + 2 * kRows - 1) / (2 * kRows);  // units per instance
    x.units = x.upi * BH;
    x.rank = rank;
    auto* bars = x.bars;

    if (tid == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->q_full[t], 1);
            mbar_init(&bars->q_free[t], 1 + 4);  // the tile's last GEMM1 + the softmax group's four warps
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 4);      // one arrival per warp of the softmax group
            mbar_init(&bars->o_full[t], 1);
            mbar_init(&bars->o_free[t], 4);      // one arrival per warp of the epilogue group
            mbar_init(&bars->den_full[t], 4);    // one arrival per warp of the softmax group
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->never, 1);
        // the operand layouts assume a 1024-byte aligned base (128-byte swizzle atoms)
        bars->abort = (x.sbase & 1023u) ? 1 : 0;
        if (x.sbase & 1023u) atomicExch(&g_device_status, 3);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&bars->tmem_base)),
                     "r"(C::tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = bars->tmem_base;
    if (force_timeout_ns) {
        // test hook: a wait on a barrier phase that nothing completes
        if (tid == 0 && !mbar_wait(&bars->never, 0, force_timeout_ns)) x.give_up();
        __syncthreads();
    }
    const bool go = *x.abort_flag == 0;
    // the preparation grid (V_S^T, w, kmax) has finished and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
        if (go && lane == 0) {
            if (warp == 0) role_producer<D>(x, &tmQ, &tmK, &tmV, wpad, rpad);
            else if (warp == 1) role_mma<D>(x);
        }
    } else if (warp < 12) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        if (go) role_softmax<D>(x, (warp - 4) >> 2, warp & 3, lane, beta, kmax);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
        if (go) role_epilogue<D>(x, warp & 3, lane, &tmO, vmin, vmax);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(x.tmem), "r"(C::tmem_cols)
                     : "memory");
    }
}

// V_S^T rounded to bf16 and w zero-padded to rpad rows, both zero at and past
// the rank: VT[b, c, l] for c < D, l < rpad; wpad[b, l].  The first block of
// each instance also forms kmax[b] = max_{l < rank} |K_S[b, l]| (the
// pivot-key half of the per-row shift).  The attend kernel that follows is
// launched as a programmatic dependent: it may start its prologue now and
// waits for this grid before it reads VT, wpad or kmax.
template <int D>
__global__ void vt_prep_kernel(const float* __restrict__ V_S, const float* __restrict__ w,
                               const __nv_bfloat16* __restrict__ K_S, const int32_t* __restrict__ rank, int r,
                               int rpad, __nv_bfloat16* __restrict__ VT, float* __restrict__ wpad,
                               float* __restrict__ kmax) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float tile[32][33];
    const int64_t b = blockIdx.z;
    const int l0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    const int rr = rank[b];
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int l = l0 + k;
        tile[k][threadIdx.x] = l < rr ? V_S[(b * r + l) * (int64_t)D + c0 + threadIdx.x] : 0.f;
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += blockDim.y)
        VT[(b * D + c0 + k) * (int64_t)rpad + l0 + threadIdx.x] = __float2bfloat16_rn(tile[threadIdx.x][k]);
    if (blockIdx.y == 0 && threadIdx.y == 0) {
        const int l = l0 + threadIdx.x;
        wpad[b * rpad + l] = l < rr ? w[b * r + l] : 0.f;
    }
    if (blockIdx.x != 0 || blockIdx.y != 0) return;  // uniform per block
    const int tid = threadIdx.y * blockDim.x + threadIdx.x, nt = blockDim.x * blockDim.y;
    float best = 0.f;
    for (int l = tid; l < rr; l += nt) {
        const uint4* k4 = reinterpret_cast<const uint4*>(K_S + (b * r + l) * D);
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            float x[8];
            load8(reinterpret_cast<const __nv_bfloat16*>(k4 + c), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(x[e], x[e], s);
        }
        best = fmaxf(best, sqrtf(s));
    }
    best = warp_max(best);
    __shared__ float wb[32];
    if ((tid & 31) == 0) wb[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
        float v = 0.f;
        for (int k = 0; k < nt / 32; ++k) v = fmaxf(v, wb[k]);
        kmax[b] = v;
    }
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

template <int D>
Status run_tc(const AttendRequest& q, void* scratch, cudaStream_t st) {
    using C = Cfg<D>;
    const int rpad = (int)round_up(q.r, kChunk);
    char* p = static_cast<char*>(scratch);
    __nv_bfloat16* VT = reinterpret_cast<__nv_bfloat16*>(p);
    p += round_up((int64_t)sizeof(__nv_bfloat16) * q.BH * D * rpad, 256);
    float* wpad = reinterpret_cast<float*>(p);
    p += round_up((int64_t)sizeof(float) * q.BH * rpad, 256);
    float* kmax = reinterpret_cast<float*>(p);
    vt_prep_kernel<D><<<dim3((unsigned)(rpad / 32), D / 32, (unsigned)q.BH), dim3(32, 8), 0, st>>>(
        q.V_S, q.w, static_cast<const __nv_bfloat16*>(q.K_S), q.rank, q.r, rpad, VT, wpad, kmax);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc: prep launch");
    if (q.m == 0) return Status::ok();
    CUtensorMap tmQ, tmK, tmV, tmO;
    const uint64_t BH = (uint64_t)q.BH, m = (uint64_t)q.m, r = (uint64_t)q.r;
    bool ok = make_tmap_3d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.Q, D, m, BH, D * 2ull, m * D * 2ull, 64, kRows) &&
              make_tmap_3d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.K_S, D, r, BH, D * 2ull, r * D * 2ull, 64,
                           kChunk) &&
              make_tmap_3d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, VT, (uint64_t)rpad, D, BH, rpad * 2ull,
                           (uint64_t)D * rpad * 2ull, 64, D) &&
              make_tmap_3d(&tmO, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, q.O, D, m, BH, D * 4ull, m * D * 4ull, 32, kRows);
    if (!ok) return Status::fail(3, "attend_tc: tensor map encoding failed");
    e = cudaFuncSetAttribute(attend_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::total);
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc: shared memory attribute");
    const int64_t units = ceil_div(q.m, 2 * kRows) * q.BH;
    if (units >= (int64_t(1) << 31)) return Status::fail(2, "attend_tc: more than 2^31 query-tile pairs");
    const unsigned grid = (unsigned)std::min<int64_t>(units, sm_count());
    // a programmatic dependent of vt_prep_kernel: its prologue overlaps the
    // preparation, and it waits for that grid before the first read of VT, wpad, kmax
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attend_tc_kernel<D>, tmQ, tmK, tmV, tmO, (const float*)wpad, rpad, (int64_t)q.m,
                           (int64_t)q.BH, q.rank, q.beta, q.vmin, q.vmax, (const float*)kmax, g_force_timeout_ns);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc launch");
    return Status::ok();
}

}  // namespace

bool attend_tc_supported(int dtype, int d) { return dtype == 1 && (d == 64 || d == 128); }

size_t attend_tc_scratch_bytes(int64_t BH, int d, int r) {
    const int64_t rpad = round_up(r, kChunk);
    return (size_t)(round_up((int64_t)sizeof(__nv_bfloat16) * BH * d * rpad, 256) +
                    round_up((int64_t)sizeof(float) * BH * rpad, 256) + (int64_t)sizeof(float) * BH);
}

Status launch_attend_tc(const AttendRequest& q, void* scratch, cudaStream_t st) {
    if ((reinterpret_cast<uintptr_t>(q.O) & 15u) || (reinterpret_cast<uintptr_t>(q.Q) & 15u) ||
        (reinterpret_cast<uintptr_t>(q.K_S) & 15u) || (reinterpret_cast<uintptr_t>(q.vmin) & 15u) ||
        (reinterpret_cast<uintptr_t>(q.vmax) & 15u))
        return Status::fail(1, "attend_tc: Q, K_S, O, vmin and vmax must be 16-byte aligned");
    switch (q.d) {
        case 64: return run_tc<64>(q, scratch, st);
        case 128: return run_tc<128>(q, scratch, st);
    }
    return Status::fail(2, "attend_tc: unsupported head dim");
}

void set_attend_force_timeout(unsigned long long ns) { g_force_timeout_ns = ns; }

int read_attend_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
    }
    return v;
}

}  // namespace wildcat
