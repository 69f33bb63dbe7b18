// weights_inverse.cu -- Nystrom weights through the maintained inverse (sm_100a, fp64).
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: RPNys
// keeps h(K_S, K_S)^-1 and grows it by a rank-one update as each pivot s
// joins S: with b = h(K_S, k_s), y = H_S^-1 b and the residual
// sc = h(k_s, k_s) - b.y,
//     H_S'^-1 = [[H_S^-1, 0], [0, 0]] + g g^T,   g = (y, -1) / sqrt(sc).
// The weights applied to (V, 1_n) are then W (V, 1_n) = H_S^-1 h(K_S, K) (V, 1_n).
// This is the same W as the factor route (weights.cu) in exact arithmetic;
// the route exists to compare the two numerically.  Its arithmetic is fp64
// throughout (the inverse amplifies rounding by the condition number of
// h(K_S, K_S), up to 1 / eps after truncation), from inputs widened exactly.
//
// Kernels (one instance b per blockIdx.y / .z):
//   knorm_partial / knorm_finalize  M_b = max_l |k_l|^2 (the shift; it cancels in W)
//   hss_kernel       H[b][a][c] = exp(beta (<k_Sa, k_Sc> - M_b)), a, c < r'
//   z_kernel         Zpart[split][b][a][:] = sum over the split's keys of
//                    exp(beta (<k_Sa, k_l> - M_b)) (v_l, 1)
//   inverse_kernel   one CTA per instance: the bordered inverse, pivot by
//                    pivot (a matrix-vector product and a rank-one update per
//                    pivot; the inverse in shared memory when it fits, else in
//                    global memory), and the sum of Zpart over splits
//   inverse_cluster_kernel  the same over a cluster of CS CTAs per instance,
//                    each holding a block of the inverse's rows in shared
//                    memory (r too large for one CTA, up to about 630)
//   xsolve_kernel    (V_S, w) = H_S^-1 Z, rounded to float32
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace wildcat {

namespace {

constexpr int kNmThreads = 256;

template <typename E, int D>
__global__ void __launch_bounds__(kNmThreads) knorm_partial(const typename E::T* K, int64_t n, int64_t rows_per_split,
                                                            double* part) {
    const int64_t b = blockIdx.y;
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int64_t l0 = split * rows_per_split, l1 = std::min<int64_t>(n, l0 + rows_per_split);
    double best = 0.0;
    for (int64_t l = l0 + threadIdx.x; l < l1; l += kNmThreads) {
        const typename E::T* k = K + (b * n + l) * D;
        double s = 0.0;
        for (int c = 0; c < D; ++c) {
            const double v = (double)E::to_float(k[c]);
            s = fma(v, v, s);
        }
        best = fmax(best, s);
    }
    for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
    __shared__ double wb[kNmThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) wb[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        double v = 0.0;
        for (int w = 0; w < kNmThreads / 32; ++w) v = fmax(v, wb[w]);
        part[b * nsplit + split] = v;
    }
}

__global__ void knorm_finalize(const double* part, int nsplit, int64_t BH, double* M) {
    const int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (b >= BH) return;
    double v = 0.0;
    for (int s = 0; s < nsplit; ++s) v = fmax(v, part[b * nsplit + s]);
    M[b] = v;
}

// ---- H_SS tile of 16 x 16 pivots ----
constexpr int kHT = 16;

template <typename E, int D>
__global__ void __launch_bounds__(kHT* kHT) hss_kernel(const typename E::T* K, const int32_t* S, const int32_t* rank,
                                                        int64_t n, int r, double beta, const double* M, double* H) {
    __shared__ double ka[kHT][D + 1], kc[kHT][D + 1];
    const int64_t b = blockIdx.z;
    const int a0 = blockIdx.y * kHT, c0 = blockIdx.x * kHT;
    const int rr = rank[b];
    const int tid = threadIdx.x;
    for (int e = tid; e < kHT * D; e += kHT * kHT) {
        const int i = e / D, c = e % D;
        const int a = a0 + i, cc = c0 + i;
        ka[i][c] = a < rr ? (double)E::to_float(K[(b * n + S[b * r + a]) * D + c]) : 0.0;
        kc[i][c] = cc < rr ? (double)E::to_float(K[(b * n + S[b * r + cc]) * D + c]) : 0.0;
    }
    __syncthreads();
    const int i = tid / kHT, j = tid % kHT;
    const int a = a0 + i, c = c0 + j;
    if (a >= r || c >= r) return;
    double v = 0.0;
    if (a < rr && c < rr) {
        double dot = 0.0;
        for (int t = 0; t < D; ++t) dot = fma(ka[i][t], kc[j][t], dot);
        v = exp(beta * (dot - M[b]));
    }
    H[(b * r + a) * (int64_t)r + c] = v;
}

// ---- Z partials: 64 pivots x (D + 1) per CTA, keys of one split in chunks of 64 ----
// Each thread forms a 4 x 4 block of (pivot, key) dot products (eight shared
// memory loads per sixteen fp64 FMAs), then a 4 pivot x D/16 column block of
// Z.  Every dot product and every Z entry is summed in key and dimension
// order, one fma at a time.
constexpr int kZThreads = 256;
constexpr int kZA = 64;
constexpr int kZL = 64;

template <int D>
struct ZSmem {
    static constexpr size_t ks = 0;                                         // double [kZA][D + 1]
    static constexpr size_t kc = ks + sizeof(double) * kZA * (D + 1);       // double [kZL][D + 1]
    static constexpr size_t vc = kc + sizeof(double) * kZL * (D + 1);       // float  [kZL][D]
    static constexpr size_t p = vc + sizeof(float) * kZL * D;               // double [kZA][kZL + 1]
    static constexpr size_t total = p + sizeof(double) * kZA * (kZL + 1);
};

template <typename E, int D>
__global__ void __launch_bounds__(kZThreads) z_kernel(const typename E::T* K, const typename E::T* V, const int32_t* S,
                                                      const int32_t* rank, int64_t n, int r, double beta,
                                                      const double* M, int64_t keys_per_split, int64_t BH,
                                                      double* Zpart) {
    using L = ZSmem<D>;
    extern __shared__ __align__(16) unsigned char sm[];
    double(*ks)[D + 1] = reinterpret_cast<double(*)[D + 1]>(sm + L::ks);
    double(*kc)[D + 1] = reinterpret_cast<double(*)[D + 1]>(sm + L::kc);
    float(*vc)[D] = reinterpret_cast<float(*)[D]>(sm + L::vc);
    double(*P)[kZL + 1] = reinterpret_cast<double(*)[kZL + 1]>(sm + L::p);
    const int64_t b = blockIdx.z;
    const int split = blockIdx.y;
    const int a0 = blockIdx.x * kZA;
    const int rr = rank[b];
    if (a0 >= rr) return;  // whole tile past the rank: its Z rows are never read
    const int tid = threadIdx.x;
    const double Mb = M[b];
    for (int e = tid; e < kZA * D; e += kZThreads) {
        const int i = e / D, c = e % D;
        const int a = a0 + i;
        ks[i][c] = a < rr ? (double)E::to_float(K[(b * n + S[b * r + a]) * D + c]) : 0.0;
    }
    const int64_t l_begin = split * keys_per_split, l_end = std::min<int64_t>(n, l_begin + keys_per_split);
    // pivots tp * 4 + u of this thread; its keys tk + 16 v (dots) and columns tk + 16 j (Z)
    const int tp = tid >> 4, tk = tid & 15;
    constexpr int CJ = D / 16;
    double acc[4][CJ];
    double accw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        accw[u] = 0.0;
#pragma unroll
        for (int j = 0; j < CJ; ++j) acc[u][j] = 0.0;
    }
    for (int64_t l0 = l_begin; l0 < l_end; l0 += kZL) {
        __syncthreads();  // the previous chunk is consumed (and the pivot keys are staged)
        for (int e = tid; e < kZL * D; e += kZThreads) {
            const int i = e / D, c = e % D;
            const int64_t l = l0 + i;
            const bool ok = l < l_end;
            kc[i][c] = ok ? (double)E::to_float(K[(b * n + l) * D + c]) : 0.0;
            vc[i][c] = ok ? E::to_float(V[(b * n + l) * D + c]) : 0.f;
        }
        __syncthreads();
        {
            double dot[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) dot[u][v] = 0.0;
#pragma unroll 4
            for (int t = 0; t < D; ++t) {
                double x[4], y[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) x[u] = ks[tp * 4 + u][t];
#pragma unroll
                for (int v = 0; v < 4; ++v) y[v] = kc[tk + 16 * v][t];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) dot[u][v] = fma(x[u], y[v], dot[u][v]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int ia = tp * 4 + u, ll = tk + 16 * v;
                    P[ia][ll] = (a0 + ia < rr && l0 + ll < l_end) ? exp(beta * (dot[u][v] - Mb)) : 0.0;
                }
        }
        __syncthreads();
        for (int ll = 0; ll < kZL; ++ll) {
            double pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) pv[u] = P[tp * 4 + u][ll];
#pragma unroll
            for (int j = 0; j < CJ; ++j) {
                const double v = (double)vc[ll][tk + 16 * j];
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u][j] = fma(pv[u], v, acc[u][j]);
            }
            if (tk == 0)
#pragma unroll
                for (int u = 0; u < 4; ++u) accw[u] += pv[u];
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int a = a0 + tp * 4 + u;
        if (a < rr) {
            double* z = Zpart + (((int64_t)split * BH + b) * r + a) * (D + 1);
#pragma unroll
            for (int j = 0; j < CJ; ++j) z[tk + 16 * j] = acc[u][j];
            if (tk == 0) z[D] = accw[u];
        }
    }
}

// ---- the bordered inverse, one CTA per instance ----
constexpr int kInvThreads = 512;
constexpr size_t kInvSmemCap = 210 * 1024;

template <bool A_SMEM>
__global__ void __launch_bounds__(kInvThreads) inverse_kernel(const double* H, const int32_t* rank, int r, int D,
                                                              int nsplit, int64_t BH, double* Ainv, double* Zpart) {
    extern __shared__ __align__(16) unsigned char sm[];
    double* bvec = reinterpret_cast<double*>(sm);  // [r]
    double* y = bvec + r;                          // [r]
    // with A_SMEM the inverse grows in shared memory ([r][r] after y) and is
    // written to global memory once at the end
    double* As = y + r;
    __shared__ double red[kInvThreads / 32];
    __shared__ double s_sc;
    const int64_t b = blockIdx.x;
    const int rr = rank[b];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kInvThreads / 32;
    const double* Hb = H + b * (int64_t)r * r;
    double* Ag = Ainv + b * (int64_t)r * r;
    double* A = A_SMEM ? As : Ag;
    for (int a = 0; a < rr; ++a) {
        // b = h(K_S[:a], k_s): row a of H (symmetric)
        for (int j = tid; j < a; j += kInvThreads) bvec[j] = Hb[(int64_t)a * r + j];
        __syncthreads();
        // y = A^-1 b, one warp per row
        for (int j = warp; j < a; j += NW) {
            double s = 0.0;
            for (int k = lane; k < a; k += 32) s = fma(A[(int64_t)j * r + k], bvec[k], s);
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) y[j] = s;
        }
        __syncthreads();
        // sc = h(k_s, k_s) - b.y
        double part = 0.0;
        for (int j = tid; j < a; j += kInvThreads) part = fma(bvec[j], y[j], part);
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) red[warp] = part;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int w = 0; w < NW; ++w) t += red[w];
            s_sc = Hb[(int64_t)a * r + a] - t;
        }
        __syncthreads();
        const double sc = s_sc;
        // A^-1 <- [[A^-1 + y y^T / sc, -y / sc], [-y^T / sc, 1 / sc]]
        for (int j = warp; j < a; j += NW) {
            const double yj = y[j] / sc;
            for (int k = lane; k < a; k += 32) A[(int64_t)j * r + k] = fma(yj, y[k], A[(int64_t)j * r + k]);
        }
        for (int j = tid; j < a; j += kInvThreads) {
            A[(int64_t)j * r + a] = -y[j] / sc;
            A[(int64_t)a * r + j] = -y[j] / sc;
        }
        if (tid == 0) A[(int64_t)a * r + a] = 1.0 / sc;
        __syncthreads();
    }
    if constexpr (A_SMEM)
        for (int64_t e = tid; e < (int64_t)rr * r; e += kInvThreads) {
            if (e % r < rr) Ag[e] = As[e];
        }
    // Z = sum of the split partials, accumulated into split 0 in split order
    const int DP = D + 1;
    for (int64_t e = tid; e < (int64_t)rr * DP; e += kInvThreads) {
        double* z0 = Zpart + (b * r) * (int64_t)DP + e;
        double s = *z0;
        for (int sp = 1; sp < nsplit; ++sp) s += Zpart[((int64_t)sp * BH + b) * r * DP + e];
        *z0 = s;
    }
}

// The bordered inverse over a cluster: CTA c keeps rows [c RB, c RB + RB) of
// A = H_S^-1 in shared memory.  Step a applies pivot a's update to its rows
// and, in the same pass over them, forms its rows of y' = A' b' for the next
// pivot (b' = row a + 1 of H), together with its part of b'.y'.  The rows of
// y' and the parts go to every CTA of the cluster (distributed shared
// memory), so after the step's cluster barrier every CTA holds all of y' and
// forms sc' = h(k_s', k_s') - b'.y' from the parts in CTA order.  y and the
// parts are double-buffered: a peer writes step a + 1's values only after
// the barrier that ends this CTA's reads of step a's.
__global__ void __launch_bounds__(kInvThreads) inverse_cluster_kernel(const double* H, const int32_t* rank, int r,
                                                                      int RB, int CS, int D, int nsplit, int64_t BH,
                                                                      double* Ainv, double* Zpart) {
    extern __shared__ __align__(16) unsigned char sm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int c = (int)cluster.block_rank();
    const int64_t b = blockIdx.x / CS;
    double* As = reinterpret_cast<double*>(sm);  // [RB][r]
    double* yb = As + (size_t)RB * r;            // [2][r]
    double* pd = yb + 2 * (size_t)r;             // [2][CS]
    __shared__ double red[kInvThreads / 32];
    constexpr int NW = kInvThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rr = b < BH ? rank[b] : 0;
    const double* Hb = H + b * (int64_t)r * r;
    const int j0 = c * RB;
    double sc = rr > 0 ? Hb[0] : 1.0;  // pivot 0: y is empty
    for (int a = 0; a < rr; ++a) {
        const double* ycur = yb + (size_t)(a & 1) * r;  // y of pivot a (rows < a)
        double* ynext = yb + (size_t)((a + 1) & 1) * r;
        double* pnext = pd + (size_t)((a + 1) & 1) * CS;
        const bool more = a + 1 < rr;
        const double* bn = Hb + (int64_t)(a + 1) * r;  // read only when more
        double wpart = 0.0;                             // lane 0: this warp's part of b'.y'
        for (int jl = warp; jl < RB; jl += NW) {
            const int j = j0 + jl;
            if (j > a) break;  // rows past pivot a do not exist yet (warp-uniform)
            double* Aj = As + (size_t)jl * r;
            double s = 0.0;
            if (j < a) {
                // A <- A + y y^T / sc on row j, then column a = -y_j / sc
                const double yj = ycur[j] / sc;
                for (int k = lane; k < a; k += 32) {
                    const double v = fma(yj, ycur[k], Aj[k]);
                    Aj[k] = v;
                    if (more) s = fma(v, bn[k], s);
                }
                if (lane == 0) {
                    const double v = -ycur[j] / sc;
                    Aj[a] = v;
                    if (more) s = fma(v, bn[a], s);
                }
            } else {
                // the new row: (-y^T / sc, 1 / sc)
                for (int k = lane; k < a; k += 32) {
                    const double v = -ycur[k] / sc;
                    Aj[k] = v;
                    if (more) s = fma(v, bn[k], s);
                }
                if (lane == 0) {
                    const double v = 1.0 / sc;
                    Aj[a] = v;
                    if (more) s = fma(v, bn[a], s);
                }
            }
            if (more) {
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane < CS) *cluster.map_shared_rank(ynext + j, lane) = s;
                if (lane == 0) wpart = fma(bn[j], s, wpart);
            }
        }
        if (more) {
            if (lane == 0) red[warp] = wpart;
            __syncthreads();
            if (tid < CS) {
                double t = 0.0;
                for (int w = 0; w < NW; ++w) t += red[w];
                *cluster.map_shared_rank(pnext + c, tid) = t;
            }
        }
        cluster.sync();
        if (more) {
            double t = 0.0;
            for (int q = 0; q < CS; ++q) t += pnext[q];
            sc = bn[a + 1] - t;
        }
    }
    if (b >= BH) return;
    double* Ag = Ainv + b * (int64_t)r * r;
    const int nown = std::max(0, std::min(RB, rr - j0));
    for (int64_t e = tid; e < (int64_t)nown * r; e += kInvThreads) {
        const int jl = (int)(e / r), k = (int)(e % r);
        if (k < rr) Ag[(int64_t)(j0 + jl) * r + k] = As[e];
    }
    // Z = sum of the split partials, accumulated into split 0 in split order
    const int DP = D + 1;
    for (int64_t e = (int64_t)c * kInvThreads + tid; e < (int64_t)rr * DP; e += (int64_t)CS * kInvThreads) {
        double* z0 = Zpart + (b * r) * (int64_t)DP + e;
        double s = *z0;
        for (int sp = 1; sp < nsplit; ++sp) s += Zpart[((int64_t)sp * BH + b) * r * DP + e];
        *z0 = s;
    }
}

// ---- (V_S, w) = A^-1 Z: 32 rows per CTA ----
constexpr int kXThreads = 256;
constexpr int kXA = 32;

template <int D>
__global__ void __launch_bounds__(kXThreads) xsolve_kernel(const double* Ainv, const double* Z, const int32_t* rank,
                                                           int r, float* V_S, float* w) {
    const int64_t b = blockIdx.y;
    const int rr = rank[b];
    const int tid = threadIdx.x;
    const int a = blockIdx.x * kXA + tid / 8, q8 = tid % 8;
    if (a >= r) return;
    constexpr int CJ = D / 8, DP = D + 1;
    double acc[CJ];
#pragma unroll
    for (int j = 0; j < CJ; ++j) acc[j] = 0.0;
    double accw = 0.0;
    if (a < rr) {
        const double* Arow = Ainv + (b * r + a) * (int64_t)r;
        const double* Zb = Z + (b * r) * (int64_t)DP;
        for (int k = 0; k < rr; ++k) {
            const double s = Arow[k];
            const double* zk = Zb + (int64_t)k * DP;
#pragma unroll
            for (int j = 0; j < CJ; ++j) acc[j] = fma(s, zk[q8 + 8 * j], acc[j]);
            accw = fma(s, zk[D], accw);
        }
    }
    float* vs = V_S + (b * r + a) * (int64_t)D;
#pragma unroll
    for (int j = 0; j < CJ; ++j) vs[q8 + 8 * j] = (float)acc[j];
    if (q8 == 0) w[b * r + a] = (float)accw;
}

// Cluster size for the shared-memory inverse: the least power of two (2..16)
// whose row blocks fit; 0 when none does.
size_t inverse_cluster_smem(int r, int CS) {
    const size_t RB = (size_t)ceil_div(r, CS);
    return sizeof(double) * (RB * r + 2 * (size_t)r + 2 * (size_t)CS);
}
int inverse_cluster_size(int r) {
    for (int cs = 2; cs <= 16; cs *= 2)
        if (inverse_cluster_smem(r, cs) <= kInvSmemCap) return cs;
    return 0;
}

struct InvPlan {
    int nsplit_m;
    int64_t rows_per_m;
    int nsplit_z;
    int64_t keys_per_split;
};

InvPlan make_inv_plan(int64_t BH, int64_t n, int r) {
    InvPlan p{};
    p.nsplit_m = (int)std::max<int64_t>(1, std::min<int64_t>(64, ceil_div(296, std::max<int64_t>(1, BH))));
    p.nsplit_m = (int)std::min<int64_t>(p.nsplit_m, std::max<int64_t>(1, n / 256));
    p.rows_per_m = ceil_div(n, p.nsplit_m);
    const int64_t tiles = ceil_div(r, kZA) * BH;
    int64_t sz = ceil_div(2 * 148, tiles);
    sz = std::max<int64_t>(1, std::min<int64_t>(sz, std::max<int64_t>(1, n / 512)));
    sz = std::min<int64_t>(sz, 64);
    p.keys_per_split = round_up(ceil_div(n, sz), kZL);
    p.nsplit_z = (int)ceil_div(n, p.keys_per_split);
    return p;
}

template <typename E, int D>
Status run_inverse(const WeightsInverseRequest& q, cudaStream_t st) {
    using T = typename E::T;
    const InvPlan p = make_inv_plan(q.BH, q.n, q.r);
    const int r = q.r;
    Carve cv(q.ws, q.ws_bytes);
    double* mpart = static_cast<double*>(cv.take(sizeof(double) * q.BH * p.nsplit_m));
    double* M = static_cast<double*>(cv.take(sizeof(double) * q.BH));
    double* H = static_cast<double*>(cv.take(sizeof(double) * q.BH * (int64_t)r * r));
    double* Ainv = static_cast<double*>(cv.take(sizeof(double) * q.BH * (int64_t)r * r));
    double* Zpart = static_cast<double*>(cv.take(sizeof(double) * p.nsplit_z * q.BH * (int64_t)r * (D + 1)));
    void* rws = cv.take(value_range_workspace_bytes(q.BH, q.n, D));
    if (!cv.fits()) return Status::fail(4, "weights_inverse: workspace too small");
    const T* K = static_cast<const T*>(q.K);
    const T* V = static_cast<const T*>(q.V);

    Status s = launch_value_range(q.V, q.dtype, q.BH, q.n, D, q.vmin, q.vmax, rws,
                                  value_range_workspace_bytes(q.BH, q.n, D), st);
    if (s.code) return s;
    knorm_partial<E, D><<<dim3(p.nsplit_m, (unsigned)q.BH), kNmThreads, 0, st>>>(K, q.n, p.rows_per_m, mpart);
    knorm_finalize<<<(unsigned)ceil_div(q.BH, 128), 128, 0, st>>>(mpart, p.nsplit_m, q.BH, M);
    const unsigned ht = (unsigned)ceil_div(r, kHT);
    hss_kernel<E, D><<<dim3(ht, ht, (unsigned)q.BH), kHT * kHT, 0, st>>>(K, q.S, q.rank, q.n, r, (double)q.beta, M,
                                                                         H);
    const size_t zsm = ZSmem<D>::total;
    cudaError_t e = cudaFuncSetAttribute(z_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)zsm);
    if (e != cudaSuccess) return Status::cuda(e, "weights_inverse: z smem attribute");
    z_kernel<E, D><<<dim3((unsigned)ceil_div(r, kZA), p.nsplit_z, (unsigned)q.BH), kZThreads, zsm, st>>>(
        K, V, q.S, q.rank, q.n, r, (double)q.beta, M, p.keys_per_split, q.BH, Zpart);
    // the inverse in shared memory: one CTA when it fits (r <= ~160), else
    // spread over a cluster (r <= ~630) while the clusters need at most about
    // two waves (then its r' sequential updates never wait on L2); else in
    // global memory, one CTA per instance in one wave.
    const bool a_sm = sizeof(double) * ((size_t)r * r + 2 * (size_t)r) <= kInvSmemCap;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int CS = a_sm ? 1 : inverse_cluster_size(r);
    if (CS > 1 && q.BH * CS > 2 * (int64_t)sms) CS = 0;
    if (CS > 1) {
        const int RB = (int)ceil_div(r, CS);
        const size_t csm = inverse_cluster_smem(r, CS);
        e = cudaFuncSetAttribute(inverse_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csm);
        if (e == cudaSuccess && CS > 8)
            e = cudaFuncSetAttribute(inverse_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return Status::cuda(e, "weights_inverse: cluster inverse attributes");
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(q.BH * CS));
        cfg.blockDim = dim3(kInvThreads);
        cfg.dynamicSmemBytes = csm;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, inverse_cluster_kernel, (const double*)H, q.rank, r, RB, CS, D, p.nsplit_z, q.BH,
                               Ainv, Zpart);
        if (e != cudaSuccess) return Status::cuda(e, "weights_inverse: cluster inverse launch");
    } else {
        const size_t ism = sizeof(double) * (2 * (size_t)r + (a_sm ? (size_t)r * r : 0));
        auto kern = a_sm ? inverse_kernel<true> : inverse_kernel<false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
        if (e != cudaSuccess) return Status::cuda(e, "weights_inverse: inverse smem attribute");
        kern<<<(unsigned)q.BH, kInvThreads, ism, st>>>(H, q.rank, r, D, p.nsplit_z, q.BH, Ainv, Zpart);
    }
    xsolve_kernel<D><<<dim3((unsigned)ceil_div(r, kXA), (unsigned)q.BH), kXThreads, 0, st>>>(Ainv, Zpart, q.rank, r,
                                                                                             q.V_S, q.w);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "weights_inverse launch");
    return Status::ok();
}

}  // namespace

size_t weights_inverse_workspace_bytes(int64_t BH, int64_t n, int d, int r) {
    const InvPlan p = make_inv_plan(BH, n, r);
    Carve cv(nullptr, 0);
    cv.take(sizeof(double) * BH * p.nsplit_m);
    cv.take(sizeof(double) * BH);
    cv.take(sizeof(double) * BH * (int64_t)r * r);
    cv.take(sizeof(double) * BH * (int64_t)r * r);
    cv.take(sizeof(double) * p.nsplit_z * BH * (int64_t)r * (d + 1));
    cv.take(value_range_workspace_bytes(BH, n, d));
    return cv.used + 256;
}

Status launch_weights_inverse(const WeightsInverseRequest& q, cudaStream_t st) {
    if (q.r > kInverseMaxRank) return Status::fail(2, "weights_inverse: r above 2048");
    const bool bf = q.dtype == 1;
    switch (q.d) {
        case 32: return bf ? run_inverse<BF16, 32>(q, st) : run_inverse<F32, 32>(q, st);
        case 64: return bf ? run_inverse<BF16, 64>(q, st) : run_inverse<F32, 64>(q, st);
        case 128: return bf ? run_inverse<BF16, 128>(q, st) : run_inverse<F32, 128>(q, st);
    }
    return Status::fail(2, "weights_inverse: unsupported head dim");
}

}  // namespace wildcat
