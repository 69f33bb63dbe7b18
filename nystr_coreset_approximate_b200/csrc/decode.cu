// decode.cu -- KV-cache decode with new tokens over a compressed cache.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: after
// CompressKV keeps (K_S, V_S = W V, w = W 1_n) of a long cache, m new tokens
// cost O(rmd + m^2 d).  New query i attends over the weighted coreset and,
// exactly, over the new tokens j <= i (causal):
//   N_i = sum_l u_il V_S,l + sum_{j<=i} e_ij v_j,   D_i = sum_l u_il w_l + sum_{j<=i} e_ij,
//   u_il = exp(beta <q_i, k_S_l> - beta M),  e_ij = exp(beta <q_i, k_j> - beta M),
// one shift M = max_i |q_i| * max(max_l |k_S_l|, max_j |k_j|) per instance,
// O_i = clip(N_i / D_i) to the value range of the cache and the new values.
//
// Kernels: decode_stats (shift and combined range, one CTA per instance) and
// decode_kernel (64 new queries per CTA, CUDA cores, fp32).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace wildcat {

namespace {

constexpr int kDecThreads = 256;
constexpr int kDecTM = 64;  // new queries per CTA
constexpr int kDecRC = 32;  // keys per chunk

template <typename E, int D>
__global__ void __launch_bounds__(kDecThreads) decode_stats(const typename E::T* Qn, const typename E::T* Kn,
                                                            const typename E::T* Vn, const typename E::T* K_S,
                                                            const int32_t* rank, const float* vmin, const float* vmax,
                                                            int64_t m, int r, float* M, float* lo, float* hi) {
    const int64_t b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = kDecThreads / 32;
    float qb = 0.f, kb = 0.f;
    for (int64_t i = warp; i < m; i += NW) {
        float sq = 0.f, sk = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float q = E::to_float(Qn[(b * m + i) * D + c]);
            const float k = E::to_float(Kn[(b * m + i) * D + c]);
            sq = fmaf(q, q, sq);
            sk = fmaf(k, k, sk);
        }
        qb = fmaxf(qb, sqrtf(warp_sum(sq)));
        kb = fmaxf(kb, sqrtf(warp_sum(sk)));
    }
    const int rr = rank[b];
    for (int l = warp; l < rr; l += NW) {
        float s = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float k = E::to_float(K_S[(b * r + l) * D + c]);
            s = fmaf(k, k, s);
        }
        kb = fmaxf(kb, sqrtf(warp_sum(s)));
    }
    __shared__ float sq_[NW], sk_[NW];
    if (lane == 0) {
        sq_[warp] = qb;
        sk_[warp] = kb;
    }
    for (int c = threadIdx.x; c < D; c += kDecThreads) {
        float l = vmin[b * D + c], h = vmax[b * D + c];
        for (int64_t j = 0; j < m; ++j) {
            const float v = E::to_float(Vn[(b * m + j) * D + c]);
            l = fminf(l, v);
            h = fmaxf(h, v);
        }
        lo[b * D + c] = l;
        hi[b * D + c] = h;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float q = 0.f, k = 0.f;
        for (int w = 0; w < NW; ++w) {
            q = fmaxf(q, sq_[w]);
            k = fmaxf(k, sk_[w]);
        }
        M[b] = q * k;
    }
}

template <typename E, int D>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const typename E::T* Qn, const typename E::T* Kn,
                                                             const typename E::T* Vn, const typename E::T* K_S,
                                                             const float* V_S, const float* w, const int32_t* rank,
                                                             int64_t m, int r, float beta, const float* M,
                                                             const float* lo, const float* hi, float* O) {
    constexpr int QS = D + 1;
    extern __shared__ __align__(16) unsigned char sm[];
    float* Qs = reinterpret_cast<float*>(sm);
    float* Ks = Qs + kDecTM * QS;
    float* Vs = Ks + kDecRC * D;
    float* ws = Vs + kDecRC * D;
    float* P = ws + kDecRC;
    const int64_t b = blockIdx.y;
    const int64_t i0 = (int64_t)blockIdx.x * kDecTM;
    const int tid = threadIdx.x;
    const int rr = rank[b];
    const float shift = beta * M[b];
    for (int e = tid; e < kDecTM * D; e += kDecThreads) {
        const int ii = e / D, c = e % D;
        const int64_t i = i0 + ii;
        Qs[ii * QS + c] = i < m ? E::to_float(Qn[(b * m + i) * D + c]) : 0.f;
    }
    constexpr int CPT = D / 4;
    const int oi = tid / 4, oc = tid % 4;
    float acc[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) acc[k] = 0.f;
    float den = 0.f;
    // the coreset rows, then the new tokens up to the tile's last query (causal)
    const int64_t jmax = std::min<int64_t>(m, i0 + kDecTM);
    const int64_t total = rr + jmax;
    for (int64_t c0 = 0; c0 < total; c0 += kDecRC) {
        __syncthreads();
        for (int e = tid; e < kDecRC * D; e += kDecThreads) {
            const int ll = e / D, c = e % D;
            const int64_t x = c0 + ll;
            float kv = 0.f, vv = 0.f;
            if (x < rr) {
                kv = E::to_float(K_S[(b * r + x) * D + c]);
                vv = V_S[(b * r + x) * (int64_t)D + c];
            } else if (x < total) {
                const int64_t j = x - rr;
                kv = E::to_float(Kn[(b * m + j) * D + c]);
                vv = E::to_float(Vn[(b * m + j) * D + c]);
            }
            Ks[ll * D + c] = kv;
            Vs[ll * D + c] = vv;
        }
        for (int ll = tid; ll < kDecRC; ll += kDecThreads) {
            const int64_t x = c0 + ll;
            ws[ll] = x < rr ? w[b * r + x] : (x < total ? 1.f : 0.f);
        }
        __syncthreads();
        for (int e = tid; e < kDecTM * kDecRC; e += kDecThreads) {
            const int ii = e % kDecTM, ll = e / kDecTM;
            const int64_t x = c0 + ll, i = i0 + ii;
            float s = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) s = fmaf(Qs[ii * QS + c], Ks[ll * D + c], s);
            const bool live = x < rr || (x < total && x - rr <= i);
            P[ii * (kDecRC + 1) + ll] = live ? expf(beta * s - shift) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ll = 0; ll < kDecRC; ++ll) {
            const float p = P[oi * (kDecRC + 1) + ll];
#pragma unroll
            for (int k = 0; k < CPT; ++k) acc[k] = fmaf(p, Vs[ll * D + oc + 4 * k], acc[k]);
            den = fmaf(p, ws[ll], den);
        }
    }
    const int64_t i = i0 + oi;
    if (i < m) {
        float* o = O + (b * m + i) * D;
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int c = oc + 4 * k;
            o[c] = fminf(fmaxf(acc[k] / den, lo[b * D + c]), hi[b * D + c]);
        }
    }
}

template <typename E, int D>
Status run_decode(const DecodeRequest& q, cudaStream_t st) {
    using T = typename E::T;
    Carve cv(q.ws, q.ws_bytes);
    float* M = static_cast<float*>(cv.take(sizeof(float) * q.BH));
    float* lo = static_cast<float*>(cv.take(sizeof(float) * q.BH * D));
    float* hi = static_cast<float*>(cv.take(sizeof(float) * q.BH * D));
    if (!cv.fits()) return Status::fail(4, "decode: workspace too small");
    const T* Qn = static_cast<const T*>(q.Qn);
    const T* Kn = static_cast<const T*>(q.Kn);
    const T* Vn = static_cast<const T*>(q.Vn);
    const T* KS = static_cast<const T*>(q.K_S);
    decode_stats<E, D><<<(unsigned)q.BH, kDecThreads, 0, st>>>(Qn, Kn, Vn, KS, q.rank, q.vmin, q.vmax, q.m, q.r, M, lo,
                                                              hi);
    const size_t smem = sizeof(float) * ((size_t)kDecTM * (D + 1) + 2 * kDecRC * D + kDecRC + kDecTM * (kDecRC + 1));
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return Status::cuda(e, "decode: smem attribute");
    decode_kernel<E, D><<<dim3((unsigned)ceil_div(q.m, kDecTM), (unsigned)q.BH), kDecThreads, smem, st>>>(
        Qn, Kn, Vn, KS, q.V_S, q.w, q.rank, q.m, q.r, q.beta, M, lo, hi, q.O);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "decode launch");
    return Status::ok();
}

}  // namespace

size_t decode_workspace_bytes(int64_t BH, int d) {
    Carve cv(nullptr, 0);
    cv.take(sizeof(float) * BH);
    cv.take(sizeof(float) * BH * d);
    cv.take(sizeof(float) * BH * d);
    return cv.used + 256;
}

Status launch_decode(const DecodeRequest& q, cudaStream_t st) {
    const bool bf = q.dtype == 1;
    switch (q.d) {
        case 32: return bf ? run_decode<BF16, 32>(q, st) : run_decode<F32, 32>(q, st);
        case 64: return bf ? run_decode<BF16, 64>(q, st) : run_decode<F32, 64>(q, st);
        case 128: return bf ? run_decode<BF16, 128>(q, st) : run_decode<F32, 128>(q, st);
    }
    return Status::fail(2, "decode: unsupported head dim");
}

}  // namespace wildcat
