// weights.cu -- Nystrom weights applied to (V, 1_n) on sm_100a.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: the
// plug-in estimator multiplies W with (V, 1_n) before the queries touch it;
// Alg. 2 CompressKV keeps V_S = W V and w = W 1_n.  With the partial
// Cholesky factor F (n x r') of the key kernel and its pivot block
// F_S = F[S, :] (lower triangular in pivot order),
//     W = h(K_S,K_S)^-1 h(K_S,K) = F_S^-T F^T,
// so (V_S, w) = F_S^-T Y with Y = F^T (V, 1_n).
//
// Kernels:
//   colrange_*   column-wise [v_min, v_max] of V (value-range clip bounds)
//   fty_kernel   Y partials: F^T (V, 1) over a slice of the keys (split-K),
//                CUDA cores (float32 values, or n % 4 != 0); bf16 values use the
//                tensor-core kernel of weights_tc.cu
//   gather_fs    F_S[a, j] = F[j, S_a] for j <= a (pivot rows of the factor)
//   trsm_warp_kernel / trsm_stream_kernel / trsm_kernel  sum the split-K
//                partials and back-substitute F_S^T X = Y (one warp per column
//                for r <= 1024, F_S read from shared memory; else blocked by 32
//                pivots)
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace wildcat {

namespace {

constexpr int kRangeThreads = 256;

template <typename E, int D>
__global__ void __launch_bounds__(kRangeThreads) colrange_partial(const typename E::T* V, int64_t n,
                                                                  int64_t rows_per_split, float* part) {
    // part [BH, nsplit, 2, D].  Each thread covers 8 consecutive columns
    // (one 16-byte load per row for bf16, two for fp32) of every RS-th row,
    // four rows in flight; the RS row slots are reduced in shared memory.
    constexpr int CPT = 8;                      // columns per thread
    constexpr int TPR = D / CPT;                // threads per row
    constexpr int RS = kRangeThreads / TPR;     // row slots
    const int64_t b = blockIdx.y;
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int c0 = (threadIdx.x % TPR) * CPT, rs = threadIdx.x / TPR;
    const int64_t l0 = split * rows_per_split, l1 = min(n, l0 + rows_per_split);
    float lo[CPT], hi[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        lo[k] = INFINITY;
        hi[k] = -INFINITY;
    }
    const typename E::T* Vb = V + b * n * D + c0;
    int64_t l = l0 + rs;
    for (; l + 3 * RS < l1; l += 4 * RS) {
        float v[4][CPT];
#pragma unroll
        for (int u = 0; u < 4; ++u) load8(Vb + (l + u * RS) * D, v[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                lo[k] = fminf(lo[k], v[u][k]);
                hi[k] = fmaxf(hi[k], v[u][k]);
            }
    }
    for (; l < l1; l += RS) {
        float v[CPT];
        load8(Vb + l * D, v);
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            lo[k] = fminf(lo[k], v[k]);
            hi[k] = fmaxf(hi[k], v[k]);
        }
    }
    __shared__ float slo[RS][D], shi[RS][D];
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        slo[rs][c0 + k] = lo[k];
        shi[rs][c0 + k] = hi[k];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kRangeThreads) {
        float a = INFINITY, z = -INFINITY;
        for (int k = 0; k < RS; ++k) {
            a = fminf(a, slo[k][c]);
            z = fmaxf(z, shi[k][c]);
        }
        float* p = part + ((b * nsplit + split) * 2) * D;
        p[c] = a;
        p[D + c] = z;
    }
}

__global__ void colrange_finalize(const float* part, int nsplit, int D, int64_t BH, float* vmin, float* vmax) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= BH * D) return;
    const int64_t b = t / D;
    const int c = (int)(t % D);
    float lo = INFINITY, hi = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
        const float* p = part + ((b * nsplit + s) * 2) * D;
        lo = fminf(lo, p[c]);
        hi = fmaxf(hi, p[D + c]);
    }
    vmin[t] = lo;
    vmax[t] = hi;
}

// ---- Y partials = F^T (V, 1) over one key slice: SIMT fp32 ----
constexpr int kFtyThreads = 256;
constexpr int kFtyTJ = 32;  // factor columns per CTA
constexpr int kFtyNK = 32;  // keys per smem stage

template <typename E, int D>
__global__ void __launch_bounds__(kFtyThreads) fty_kernel(const float* F, const typename E::T* V, int64_t n,
                                                          int r, int64_t keys_per_split, float* Ypart,
                                                          int64_t BH, const int32_t* rank) {
    // Ypart [nsplit, BH, r, D + 1]; rows at or past the instance's rank are
    // never read by the solve, so tiles that start there do no work.
    const int jt = blockIdx.x, split = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int j0 = jt * kFtyTJ;
    if (j0 >= rank[b]) return;
    const int64_t l0 = split * keys_per_split, l1 = min(n, l0 + keys_per_split);
    constexpr int TPR = kFtyThreads / kFtyTJ;  // threads per factor column
    constexpr int CPT = D / TPR;               // value columns per thread
    const int jj = threadIdx.x / TPR, tx = threadIdx.x % TPR;

    __shared__ float Fs[kFtyTJ][kFtyNK + 1];
    __shared__ __align__(16) float Vs[kFtyNK][D];
    float acc[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) acc[k] = 0.f;
    float one = 0.f;
    const float* Fb = F + b * (int64_t)r * n;
    const typename E::T* Vb = V + b * n * D;
    for (int64_t lb = l0; lb < l1; lb += kFtyNK) {
        for (int e = threadIdx.x; e < kFtyTJ * kFtyNK; e += kFtyThreads) {
            const int rj = e / kFtyNK, kk = e % kFtyNK;
            const int64_t l = lb + kk;
            const int j = j0 + rj;
            Fs[rj][kk] = (j < r && l < l1) ? __ldcg(Fb + (int64_t)j * n + l) : 0.f;
        }
        for (int e = threadIdx.x; e < kFtyNK * D; e += kFtyThreads) {
            const int kk = e / D, c = e % D;
            const int64_t l = lb + kk;
            Vs[kk][c] = l < l1 ? E::to_float(Vb[l * D + c]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kFtyNK; ++kk) {
            const float f = Fs[jj][kk];
#pragma unroll
            for (int k = 0; k < CPT; ++k) acc[k] = fmaf(f, Vs[kk][tx + TPR * k], acc[k]);
            one += f;
        }
        __syncthreads();
    }
    const int j = j0 + jj;
    if (j < r) {
        float* y = Ypart + (((int64_t)split * BH + b) * r + j) * (D + 1);
#pragma unroll
        for (int k = 0; k < CPT; ++k) y[tx + TPR * k] = acc[k];
        if (tx == 0) y[D] = one;
    }
}

// F_S[b, a, j] = F[b, j, S[b, a]] for j <= a < rank (the solve reads nothing else).
__global__ void gather_fs(const float* F, const int32_t* S, const int32_t* rank, int64_t n, int r, float* FS) {
    const int64_t b = blockIdx.y;
    const int a = blockIdx.x;
    const int rr = rank[b];
    if (a >= rr) return;  // the solve reads rows below the rank only
    float* dst = FS + (b * r + a) * (int64_t)r;
    const int s = S[b * r + a];
    for (int j = threadIdx.x; j <= a; j += blockDim.x) dst[j] = __ldcg(F + (b * r + j) * n + s);
}

// Back substitution F_S^T X = Y for one instance and one block of CB
// right-hand columns, blocked by 32 pivots, right-looking: blocks are solved
// bottom up; one half-warp solves a 32 x 32 diagonal block from shared
// memory (one lane per column), then all threads subtract the solved rows
// from every row above the block, reading rows of F_S contiguously.  Two
// block barriers per 32 pivots.
constexpr int kTrsmThreads = 256;
constexpr int kTrsmCB = 16;
constexpr int kTrsmBlk = 32;

__global__ void __launch_bounds__(kTrsmThreads) trsm_kernel(const float* Ypart, int nsplit, const float* FS,
                                                            const int32_t* rank, int64_t BH, int r, int D,
                                                            float* V_S, float* w) {
    extern __shared__ float X[];  // [r][CB], then the diagonal block [32][33]
    float* Ld = X + (size_t)r * kTrsmCB;
    constexpr int LDS = kTrsmBlk + 1;
    const int64_t b = blockIdx.y;
    const int cb0 = blockIdx.x * kTrsmCB;
    const int DP = D + 1;
    const int rr = rank[b];
    const int c = threadIdx.x % kTrsmCB, rs = threadIdx.x / kTrsmCB;
    constexpr int RS = kTrsmThreads / kTrsmCB;
    const int col = cb0 + c;
    const float* Lb = FS + b * (int64_t)r * r;  // Lb[a' * r + a] = F_S[a', a], a <= a'
    // diagonal block of pivots [a0, a0 + nb): Ld[i][j] = F_S[a0 + i, a0 + j], j <= i
    auto stage_diag = [&](int a0, int nb) {
        for (int e = threadIdx.x; e < kTrsmBlk * kTrsmBlk; e += kTrsmThreads) {
            const int i = e / kTrsmBlk, j = e % kTrsmBlk;
            Ld[i * LDS + j] = (i < nb && j <= i) ? Lb[(int64_t)(a0 + i) * r + a0 + j] : 0.f;
        }
    };
    for (int a = rs; a < r; a += RS) {
        float y = 0.f;
        if (a < rr && col < DP)
            for (int s = 0; s < nsplit; ++s) y += Ypart[(((int64_t)s * BH + b) * r + a) * DP + col];
        X[a * kTrsmCB + c] = y;
    }
    const int nblk = (rr + kTrsmBlk - 1) / kTrsmBlk;
    if (nblk > 0) {
        const int a0 = (nblk - 1) * kTrsmBlk;
        stage_diag(a0, rr - a0);
    }
    __syncthreads();
    for (int blk = nblk - 1; blk >= 0; --blk) {
        const int a0 = blk * kTrsmBlk, nb = min(rr, a0 + kTrsmBlk) - a0;
        // (1) the diagonal block, bottom up, one lane per right-hand column
        if (threadIdx.x < kTrsmCB) {
            for (int i = nb - 1; i >= 0; --i) {
                const float xa = X[(a0 + i) * kTrsmCB + c] / Ld[i * LDS + i];
                X[(a0 + i) * kTrsmCB + c] = xa;
                for (int j = 0; j < i; ++j)
                    X[(a0 + j) * kTrsmCB + c] = fmaf(-Ld[i * LDS + j], xa, X[(a0 + j) * kTrsmCB + c]);
            }
        }
        __syncthreads();
        // (2) rows above the block: X[a] -= sum_i F_S[a0 + i, a] X[a0 + i]; stage the next diagonal block
        for (int a = rs; a < a0; a += RS) {
            float acc = X[a * kTrsmCB + c];
            const float* Lcol = Lb + (int64_t)a0 * r + a;
            for (int i = 0; i < nb; ++i) acc = fmaf(-Lcol[(int64_t)i * r], X[(a0 + i) * kTrsmCB + c], acc);
            X[a * kTrsmCB + c] = acc;
        }
        if (blk > 0) stage_diag(a0 - kTrsmBlk, kTrsmBlk);
        __syncthreads();
    }
    if (col < DP) {
        for (int a = rs; a < r; a += RS) {
            const float v = a < rr ? X[a * kTrsmCB + c] : 0.f;
            if (col < D)
                V_S[(b * r + a) * (int64_t)D + col] = v;
            else
                w[b * r + a] = v;
        }
    }
}

// Back substitution with one warp per right-hand column (r <= kTrsmWarpMaxR),
// kTrsmWarps columns per CTA.  The CTA sums the split-K partials of its
// columns (coalesced over the columns); F_S is then read from shared memory,
// copied whole when it fits (r <= ~220), else streamed a sub-block of pivots
// at a time.  Pivot a (bottom up) gives x_a = y_a / F_S[a, a], and the lanes
// subtract F_S[a, j] x_a from every y_j, j < a, reading row a contiguously;
// lane l holds y[32 m + l] in registers.
constexpr int kTrsmWarps = 8;
constexpr int kTrsmWarpMaxR = 1024;
constexpr int kTrsmRegs = kTrsmWarpMaxR / 32;  // y values per lane
constexpr size_t kTrsmSmemCap = 200 * 1024;

inline bool trsm_fs_in_smem(int r) {
    return sizeof(float) * ((size_t)kTrsmWarps * r + (size_t)r * r) <= kTrsmSmemCap;
}

// cp.async helpers (global -> shared, L2 only for 16 bytes)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Sum of the split-K partials of the CTA's kTrsmWarps columns, coalesced over
// the columns: ysm[c][j] = sum_sp Ypart[sp][b][j][cb0 + c] for j < rr.
__device__ __forceinline__ void trsm_sum_partials(const float* __restrict__ Ypart, int nsplit, int64_t BH, int64_t b,
                                                  int r, int rr, int DP, int cb0, float* ysm) {
#pragma unroll 4
    for (int e = threadIdx.x; e < rr * kTrsmWarps; e += kTrsmWarps * 32) {
        const int j = e / kTrsmWarps, c = e % kTrsmWarps;
        float s = 0.f;
        if (cb0 + c < DP) {
            const float* src = Ypart + ((int64_t)b * r + j) * DP + cb0 + c;
            const int64_t stride = BH * (int64_t)r * DP;
#pragma unroll 8
            for (int sp = 0; sp < nsplit; ++sp) s += src[sp * stride];
        }
        ysm[(size_t)c * r + j] = s;
    }
}

// Writes column `col` of (V_S | w) from the registers of the warp's solve.
__device__ __forceinline__ void trsm_store(const float (&yr)[kTrsmRegs], int lane, int64_t b, int r, int rr, int D,
                                           int col, float* V_S, float* w) {
#pragma unroll
    for (int m = 0; m < kTrsmRegs; ++m) {
        const int j = 32 * m + lane;
        if (j >= r) break;
        const float v = j < rr ? yr[m] : 0.f;
        if (col < D)
            V_S[(b * r + j) * (int64_t)D + col] = v;
        else
            w[b * r + j] = v;
    }
}

// Pivot a of the back substitution, from row a of F_S (La[j] = F_S[a, j]):
// x_a = y_a / F_S[a, a] (y_a broadcast from its lane), then y_j -= F_S[a, j] x_a
// for every j < a.  Called from loops over the register block MB = a / 32
// that are unrolled, so every register index is static.
__device__ __forceinline__ void trsm_pivot(float (&yr)[kTrsmRegs], const float* La, int a, int MB, int lane) {
    const int la = a - 32 * MB;
    const float ya = __shfl_sync(0xffffffffu, yr[MB], la);
    const float xa = ya / La[a];
#pragma unroll
    for (int m = 0; m < MB; ++m) yr[m] = fmaf(-La[32 * m + lane], xa, yr[m]);
    if (lane < la) yr[MB] = fmaf(-La[32 * MB + lane], xa, yr[MB]);
    if (lane == la) yr[MB] = xa;
}

// F_S in shared memory as a whole (small r): the CTA sums its columns'
// partials and copies F_S (16-byte loads, eight in flight per thread), then
// each warp solves its column with every row read on chip.
__global__ void __launch_bounds__(kTrsmWarps * 32) trsm_warp_kernel(const float* __restrict__ Ypart, int nsplit,
                                                                    const float* __restrict__ FS,
                                                                    const int32_t* rank, int64_t BH, int r, int D,
                                                                    float* V_S, float* w) {
    extern __shared__ float ysm[];  // [kTrsmWarps][r], then F_S [r][r]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int cb0 = blockIdx.x * kTrsmWarps;
    const int DP = D + 1;
    const int rr = rank[b];
    const int col = cb0 + warp;
    const float* __restrict__ Lg = FS + b * (int64_t)r * r;  // Lg[a * r + j] = F_S[a, j], j <= a
    float* Ls = ysm + (size_t)kTrsmWarps * r;
    trsm_sum_partials(Ypart, nsplit, BH, b, r, rr, DP, cb0, ysm);
    if ((r & 3) == 0) {
        const int q4 = r >> 2;
#pragma unroll 8
        for (int e = threadIdx.x; e < rr * q4; e += kTrsmWarps * 32) {
            const int a = e / q4, j = (e % q4) * 4;
            float4 v = __ldg(reinterpret_cast<const float4*>(Lg) + e);
            if (j + 0 > a) v.x = 0.f;
            if (j + 1 > a) v.y = 0.f;
            if (j + 2 > a) v.z = 0.f;
            if (j + 3 > a) v.w = 0.f;
            reinterpret_cast<float4*>(Ls)[e] = v;
        }
    } else {
#pragma unroll 8
        for (int e = threadIdx.x; e < rr * r; e += kTrsmWarps * 32) {
            const int a = e / r, j = e % r;
            Ls[e] = j <= a ? Lg[e] : 0.f;
        }
    }
    __syncthreads();
    if (col >= DP) return;  // no block-wide synchronisation below
    const float* y = ysm + (size_t)warp * r;
    float yr[kTrsmRegs];
#pragma unroll
    for (int m = 0; m < kTrsmRegs; ++m) {
        const int j = 32 * m + lane;
        yr[m] = j < rr ? y[j] : 0.f;
    }
#pragma unroll
    for (int mb = kTrsmRegs - 1; mb >= 0; --mb) {
        if (32 * mb >= rr) continue;
        const int top = min(31, rr - 1 - 32 * mb);
        for (int la = top; la >= 0; --la) {
            const int a = 32 * mb + la;
            trsm_pivot(yr, Ls + (int64_t)a * r, a, mb, lane);
        }
    }
    trsm_store(yr, lane, b, r, rr, D, col, V_S, w);
}

// F_S streamed through shared memory (larger r): rows are staged R at a time
// (the R pivots of one sub-block, bottom up; only the columns j < 32 (a/32 + 1)
// the sweep reads), double-buffered with cp.async, so every warp of the CTA
// reads the rows on chip and the copy of the next sub-block runs while this
// one is applied.  The same arithmetic per pivot as the kernel above.
template <int R>
__global__ void __launch_bounds__(kTrsmWarps * 32, 1) trsm_stream_kernel(const float* __restrict__ Ypart, int nsplit,
                                                                      const float* __restrict__ FS,
                                                                      const int32_t* rank, int64_t BH, int r, int D,
                                                                      float* V_S, float* w) {
    static_assert(R == 16 || R == 32, "sub-block of 16 or 32 pivots");
    extern __shared__ float ysm[];  // [kTrsmWarps][r], then two buffers of R rows of r floats
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int cb0 = blockIdx.x * kTrsmWarps;
    const int DP = D + 1;
    const int rr = rank[b];
    const int col = cb0 + warp;
    const bool active = col < DP;
    const float* __restrict__ Lg = FS + b * (int64_t)r * r;
    float* const buf0 = ysm + (size_t)kTrsmWarps * r;  // buffer k at buf0 + k * R * r
    if (rr == 0) {
        if (active) {
            float yz[kTrsmRegs];
#pragma unroll
            for (int m = 0; m < kTrsmRegs; ++m) yz[m] = 0.f;
            trsm_store(yz, lane, b, r, rr, D, col, V_S, w);
        }
        return;
    }
    const bool vec = (r & 3) == 0;
    // copy of sub-block q: rows [qR, min(qR + R, rr)), columns [0, 32 (qR / 32 + 1))
    auto issue = [&](int q) {
        float* dst = buf0 + (size_t)(q & 1) * R * r;
        const int a0 = q * R, a1 = min(a0 + R, rr);
        const int cols = min(32 * (a0 / 32 + 1), r);
        if (vec) {
            const int c4 = cols >> 2;
            for (int e = threadIdx.x; e < (a1 - a0) * c4; e += kTrsmWarps * 32) {
                const int i = e / c4, j = (e % c4) * 4;
                cp_async16(dst + (size_t)i * r + j, Lg + (int64_t)(a0 + i) * r + j);
            }
        } else {
            for (int e = threadIdx.x; e < (a1 - a0) * cols; e += kTrsmWarps * 32) {
                const int i = e / cols, j = e % cols;
                cp_async4(dst + (size_t)i * r + j, Lg + (int64_t)(a0 + i) * r + j);
            }
        }
    };
    const int q_top = (rr - 1) / R;
    issue(q_top);
    cp_async_commit();
    trsm_sum_partials(Ypart, nsplit, BH, b, r, rr, DP, cb0, ysm);
    __syncthreads();
    float yr[kTrsmRegs];
    {
        const float* y = ysm + (size_t)warp * r;
#pragma unroll
        for (int m = 0; m < kTrsmRegs; ++m) {
            const int j = 32 * m + lane;
            yr[m] = j < rr ? y[j] : 0.f;
        }
    }
#pragma unroll
    for (int mb = kTrsmRegs - 1; mb >= 0; --mb) {
        if (32 * mb >= rr) continue;
#pragma unroll
        for (int h = 32 / R - 1; h >= 0; --h) {
            const int q = mb * (32 / R) + h;
            if (q > q_top) continue;
            if (q >= 1) issue(q - 1);
            cp_async_commit();
            cp_async_wait1();  // this thread's copies of sub-block q have landed
            __syncthreads();   // and everyone's
            if (active) {
                const float* B = buf0 + (size_t)(q & 1) * R * r;
                for (int a = min(q * R + R - 1, rr - 1); a >= q * R; --a) trsm_pivot(yr, B + (size_t)(a - q * R) * r, a, mb, lane);
            }
            __syncthreads();  // the buffer is read before the copy two sub-blocks on refills it
        }
    }
    if (active) trsm_store(yr, lane, b, r, rr, D, col, V_S, w);
}

// rows per staged sub-block: 32 while two buffers of 32 rows fit in 160 KB, else 16
inline int trsm_stream_rows(int r) { return 2 * 32 * (size_t)r * sizeof(float) <= 160 * 1024 ? 32 : 16; }
inline size_t trsm_stream_smem(int r) {
    return sizeof(float) * ((size_t)kTrsmWarps * r + 2 * (size_t)trsm_stream_rows(r) * r);
}

struct WeightsPlan {
    int nsplit_range;
    int64_t rows_per_range;
    int nsplit_k;            // split-K of the CUDA-core F^T (V, 1)
    int64_t keys_per_split;
    int nsplit_tc;           // split-K of the tensor-core F^T (V, 1)
    int64_t keys_per_split_tc;
    int max_split() const { return nsplit_k > nsplit_tc ? nsplit_k : nsplit_tc; }
};

int sm_count_or_default() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}

WeightsPlan make_plan(int64_t BH, int64_t n, int d, int r) {
    WeightsPlan p{};
    p.nsplit_range = (int)std::max<int64_t>(1, std::min<int64_t>(64, ceil_div(296, std::max<int64_t>(1, BH))));
    p.nsplit_range = (int)std::min<int64_t>(p.nsplit_range, std::max<int64_t>(1, n / 64));
    p.rows_per_range = ceil_div(n, p.nsplit_range);
    const int64_t tiles = ceil_div(r, kFtyTJ) * BH;
    int64_t sk = ceil_div(2 * 148, tiles);
    sk = std::max<int64_t>(1, std::min<int64_t>(sk, std::max<int64_t>(1, n / 256)));
    sk = std::min<int64_t>(sk, 64);
    p.keys_per_split = round_up(ceil_div(n, sk), kFtyNK);
    p.nsplit_k = (int)ceil_div(n, p.keys_per_split);
    // tensor-core tiles cover 128 factor columns (weights_tc.cu chooses the key splits)
    p.keys_per_split_tc = weights_tc_keys_per_split(BH, n, d, r, sm_count_or_default());
    p.nsplit_tc = (int)ceil_div(n, p.keys_per_split_tc);
    return p;
}

template <typename E, int D>
Status run_weights(const WeightsRequest& q, cudaStream_t st) {
    const WeightsPlan p = make_plan(q.BH, q.n, D, q.r);
    Carve cv(q.ws, q.ws_bytes);
    float* part = static_cast<float*>(cv.take(sizeof(float) * q.BH * p.nsplit_range * 2 * D));
    float* Ypart = static_cast<float*>(cv.take(sizeof(float) * p.max_split() * q.BH * (int64_t)q.r * (D + 1)));
    float* FS = static_cast<float*>(cv.take(sizeof(float) * q.BH * (int64_t)q.r * q.r));
    if (!cv.fits()) return Status::fail(4, "weights: workspace too small");
    using T = typename E::T;
    const T* V = static_cast<const T*>(q.V);

    if (!q.skip_range) {
        colrange_partial<E, D><<<dim3(p.nsplit_range, (unsigned)q.BH), kRangeThreads, 0, st>>>(V, q.n,
                                                                                               p.rows_per_range, part);
        colrange_finalize<<<(unsigned)ceil_div(q.BH * D, 256), 256, 0, st>>>(part, p.nsplit_range, D, q.BH, q.vmin,
                                                                              q.vmax);
    }
    int nsplit = p.nsplit_k;
    if (weights_tc_supported(q.dtype, D, q.n)) {
        nsplit = p.nsplit_tc;
        const Status s = launch_weights_tc(q.F, q.V, q.rank, q.BH, q.n, D, q.r, p.nsplit_tc, p.keys_per_split_tc, Ypart,
                                           st);
        if (s.code) return s;
    } else {
        fty_kernel<E, D><<<dim3((unsigned)ceil_div(q.r, kFtyTJ), p.nsplit_k, (unsigned)q.BH), kFtyThreads, 0, st>>>(
            q.F, V, q.n, q.r, p.keys_per_split, Ypart, q.BH, q.rank);
    }
    gather_fs<<<dim3(q.r, (unsigned)q.BH), 128, 0, st>>>(q.F, q.S, q.rank, q.n, q.r, FS);
    cudaError_t e;
    if (q.r <= kTrsmWarpMaxR) {
        const bool fs_sm = trsm_fs_in_smem(q.r);
        const size_t smem = fs_sm ? sizeof(float) * ((size_t)kTrsmWarps * q.r + (size_t)q.r * q.r)
                                  : trsm_stream_smem(q.r);
        auto kern = fs_sm ? trsm_warp_kernel
                          : (trsm_stream_rows(q.r) == 32 ? trsm_stream_kernel<32> : trsm_stream_kernel<16>);
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return Status::cuda(e, "weights: trsm smem attribute");
        kern<<<dim3((unsigned)ceil_div(D + 1, kTrsmWarps), (unsigned)q.BH), kTrsmWarps * 32, smem, st>>>(
            Ypart, nsplit, FS, q.rank, q.BH, q.r, D, q.V_S, q.w);
    } else {
        const size_t smem = sizeof(float) * ((size_t)q.r * kTrsmCB + kTrsmBlk * (kTrsmBlk + 1));
        e = cudaFuncSetAttribute(trsm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return Status::cuda(e, "weights: trsm smem attribute");
        trsm_kernel<<<dim3((unsigned)ceil_div(D + 1, kTrsmCB), (unsigned)q.BH), kTrsmThreads, smem, st>>>(
            Ypart, nsplit, FS, q.rank, q.BH, q.r, D, q.V_S, q.w);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "weights launch");
    return Status::ok();
}

}  // namespace

size_t weights_workspace_bytes(int64_t BH, int64_t n, int d, int r) {
    const WeightsPlan p = make_plan(BH, n, d, r);
    Carve cv(nullptr, 0);
    cv.take(sizeof(float) * BH * p.nsplit_range * 2 * d);
    cv.take(sizeof(float) * p.max_split() * BH * (int64_t)r * (d + 1));
    cv.take(sizeof(float) * BH * (int64_t)r * r);
    return cv.used + 256;
}

size_t value_range_workspace_bytes(int64_t BH, int64_t n, int d) {
    const WeightsPlan p = make_plan(BH, n, d, 1);
    return sizeof(float) * BH * p.nsplit_range * 2 * d + 256;
}

Status launch_value_range(const void* V, int dtype, int64_t BH, int64_t n, int d, float* vmin, float* vmax,
                          void* ws, size_t ws_bytes, cudaStream_t st) {
    const WeightsPlan p = make_plan(BH, n, d, 1);
    Carve cv(ws, ws_bytes);
    float* part = static_cast<float*>(cv.take(sizeof(float) * BH * p.nsplit_range * 2 * d));
    if (!cv.fits()) return Status::fail(4, "value range: workspace too small");
    const dim3 grid(p.nsplit_range, (unsigned)BH);
    const bool bf = dtype == 1;
    switch (d) {
        case 32:
            if (bf) colrange_partial<BF16, 32><<<grid, kRangeThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(V), n, p.rows_per_range, part);
            else colrange_partial<F32, 32><<<grid, kRangeThreads, 0, st>>>(static_cast<const float*>(V), n, p.rows_per_range, part);
            break;
        case 64:
            if (bf) colrange_partial<BF16, 64><<<grid, kRangeThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(V), n, p.rows_per_range, part);
            else colrange_partial<F32, 64><<<grid, kRangeThreads, 0, st>>>(static_cast<const float*>(V), n, p.rows_per_range, part);
            break;
        case 128:
            if (bf) colrange_partial<BF16, 128><<<grid, kRangeThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(V), n, p.rows_per_range, part);
            else colrange_partial<F32, 128><<<grid, kRangeThreads, 0, st>>>(static_cast<const float*>(V), n, p.rows_per_range, part);
            break;
        default: return Status::fail(2, "value range: unsupported head dim");
    }
    colrange_finalize<<<(unsigned)ceil_div(BH * d, 256), 256, 0, st>>>(part, p.nsplit_range, d, BH, vmin, vmax);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "value range launch");
    return Status::ok();
}

Status launch_weights(const WeightsRequest& q, cudaStream_t st) {
    if (((size_t)q.r * kTrsmCB + kTrsmBlk * (kTrsmBlk + 1)) * sizeof(float) > 227 * 1024)
        return Status::fail(2, "weights: r too large for the on-chip triangular solve");
    const bool bf = q.dtype == 1;
    switch (q.d) {
        case 32: return bf ? run_weights<BF16, 32>(q, st) : run_weights<F32, 32>(q, st);
        case 64: return bf ? run_weights<BF16, 64>(q, st) : run_weights<F32, 64>(q, st);
        case 128: return bf ? run_weights<BF16, 128>(q, st) : run_weights<F32, 128>(q, st);
    }
    return Status::fail(2, "weights: unsupported head dim");
}

}  // namespace wildcat
