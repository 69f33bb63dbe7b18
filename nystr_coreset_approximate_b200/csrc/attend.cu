// attend.cu -- weighted-coreset attention on sm_100a.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2 plug-in
// estimator and Alg. 3 WtdAttn: with U = exp(beta Q K_S^T),
//     O_hat = diag(U w)^-1 U V_S,  each entry clipped to [v_min j, v_max j].
// A single shift M_Q = max_i |q_i| * max_l |k_S_l| per instance keeps every
// exponent <= 0 and cancels in the ratio.
//
// Kernels:
//   qnorm_partial / shift_finalize   M_Q per instance
//   attend_kernel                    per tile of queries: P = exp(beta Q K_S^T
//                                    - beta M_Q) chunk by chunk, N += P V_S,
//                                    D += P w, then O = clip(N / D)
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace wildcat {

namespace {

constexpr int kNormThreads = 256;

template <typename E, int D>
__global__ void __launch_bounds__(kNormThreads) qnorm_partial(const typename E::T* Q, int64_t m,
                                                              int64_t rows_per_split, float* part) {
    // part [BH, nsplit]: max |q_i| over a slice of the queries; one thread
    // per row with independent 16-byte loads (no per-row reduction chain)
    const int64_t b = blockIdx.y;
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t i0 = split * rows_per_split, i1 = std::min<int64_t>(m, i0 + rows_per_split);
    float best = 0.f;
    for (int64_t i = i0 + threadIdx.x; i < i1; i += kNormThreads) {
        const typename E::T* q = Q + (b * m + i) * D;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
            float v[8];
            load8(q + c, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(v[e], v[e], s);
        }
        best = fmaxf(best, sqrtf(s));
    }
    best = warp_max(best);
    __shared__ float wb[kNormThreads / 32];
    if (lane == 0) wb[warp] = best;
    __syncthreads();
    if (warp == 0) {
        float v = lane < kNormThreads / 32 ? wb[lane] : 0.f;
        v = warp_max(v);
        if (lane == 0) part[b * nsplit + split] = v;
    }
}

template <typename E, int D>
__global__ void shift_finalize(const float* part, int nsplit, const typename E::T* K_S, const int32_t* rank, int r,
                               float* MQ) {
    const int64_t b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int rr = rank[b];
    // one pivot row per thread, read as 16-byte pieces that are all in flight
    // at once (the rows of an instance are contiguous: 16-byte aligned when
    // D * sizeof(T) is a multiple of 16, which holds for every D here)
    using T = typename E::T;
    constexpr int EP = 16 / (int)sizeof(T);  // elements per 16-byte piece
    float kb = 0.f;
    for (int l = threadIdx.x; l < rr; l += blockDim.x) {
        const uint4* k4 = reinterpret_cast<const uint4*>(K_S + (b * r + l) * D);
        uint4 pc[D / EP];
#pragma unroll
        for (int c = 0; c < D / EP; ++c) pc[c] = __ldg(k4 + c);
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < D / EP; ++c) {
            const T* e = reinterpret_cast<const T*>(&pc[c]);
#pragma unroll
            for (int q = 0; q < EP; ++q) {
                const float v = E::to_float(e[q]);
                s = fmaf(v, v, s);
            }
        }
        kb = fmaxf(kb, sqrtf(s));
    }
    kb = warp_max(kb);
    float qb = 0.f;
    for (int s = lane; s < nsplit; s += 32) qb = fmaxf(qb, part[b * nsplit + s]);
    qb = warp_max(qb);
    __shared__ float wk[32];
    if (lane == 0) wk[warp] = kb;
    __syncthreads();
    if (threadIdx.x == 0) {
        float k = 0.f;
        for (int w = 0; w < nw; ++w) k = fmaxf(k, wk[w]);
        MQ[b] = qb * k;
    }
}

constexpr int kAttThreads = 256;
constexpr int kAttTM = 64;  // queries per CTA
constexpr int kAttRC = 32;  // coreset rows per chunk

template <int D>
struct AttSmem {
    static constexpr int QS = D + 1;  // padded row stride (bank-conflict free)
    static constexpr size_t q = 0;
    static constexpr size_t k = q + sizeof(float) * kAttTM * QS;
    static constexpr size_t v = k + sizeof(float) * kAttRC * D;
    static constexpr size_t wv = v + sizeof(float) * kAttRC * D;
    static constexpr size_t p = wv + sizeof(float) * kAttRC;
    static constexpr size_t total = p + sizeof(float) * kAttTM * (kAttRC + 1);
};

template <typename E, int D>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(const typename E::T* Q, const typename E::T* K_S,
                                                             int64_t m, int r, const int32_t* rank, float beta,
                                                             const float* V_S, const float* w, const float* vmin,
                                                             const float* vmax, const float* MQ, float* O) {
    using L = AttSmem<D>;
    extern __shared__ __align__(16) unsigned char sm[];
    float* Qs = reinterpret_cast<float*>(sm + L::q);
    float* Ks = reinterpret_cast<float*>(sm + L::k);
    float* Vs = reinterpret_cast<float*>(sm + L::v);
    float* ws = reinterpret_cast<float*>(sm + L::wv);
    float* P = reinterpret_cast<float*>(sm + L::p);

    const int64_t b = blockIdx.y;
    const int64_t i0 = (int64_t)blockIdx.x * kAttTM;
    const int tid = threadIdx.x;
    const int rr = rank[b];
    const float shift = beta * MQ[b];

    for (int e = tid; e < kAttTM * D; e += kAttThreads) {
        const int ii = e / D, c = e % D;
        const int64_t i = i0 + ii;
        Qs[ii * L::QS + c] = i < m ? E::to_float(Q[(b * m + i) * D + c]) : 0.f;
    }
    constexpr int CPT = D / 4;  // output columns per thread
    const int oi = tid / 4, oc = tid % 4;
    float acc[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) acc[k] = 0.f;
    float den = 0.f;

    for (int l0 = 0; l0 < rr; l0 += kAttRC) {
        __syncthreads();  // previous chunk fully consumed (and Q tile loaded)
        for (int e = tid; e < kAttRC * D; e += kAttThreads) {
            const int ll = e / D, c = e % D;
            const int l = l0 + ll;
            const bool ok = l < rr;
            Ks[ll * D + c] = ok ? E::to_float(K_S[(b * r + l) * D + c]) : 0.f;
            Vs[ll * D + c] = ok ? V_S[(b * r + l) * (int64_t)D + c] : 0.f;
        }
        for (int ll = tid; ll < kAttRC; ll += kAttThreads) ws[ll] = (l0 + ll < rr) ? w[b * r + l0 + ll] : 0.f;
        __syncthreads();
        // P[i][l] = exp(beta <q_i, k_l> - beta M_Q), zero past the rank
        for (int e = tid; e < kAttTM * kAttRC; e += kAttThreads) {
            const int ii = e % kAttTM, ll = e / kAttTM;
            float s = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) s = fmaf(Qs[ii * L::QS + c], Ks[ll * D + c], s);
            P[ii * (kAttRC + 1) + ll] = (l0 + ll < rr) ? expf(beta * s - shift) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ll = 0; ll < kAttRC; ++ll) {
            const float p = P[oi * (kAttRC + 1) + ll];
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
            o[c] = fminf(fmaxf(acc[k] / den, vmin[b * D + c]), vmax[b * D + c]);
        }
    }
}

template <typename E, int D>
Status run_attend(const AttendRequest& q, cudaStream_t st) {
    using T = typename E::T;
    const int nsplit = (int)std::max<int64_t>(1, std::min<int64_t>(64, ceil_div(q.m, 1024)));
    const int64_t rows_per_split = ceil_div(q.m, nsplit);
    Carve cv(q.ws, q.ws_bytes);
    float* part = static_cast<float*>(cv.take(sizeof(float) * q.BH * nsplit));
    float* MQ = static_cast<float*>(cv.take(sizeof(float) * q.BH));
    if (!cv.fits()) return Status::fail(4, "attend: workspace too small");
    const T* Q = static_cast<const T*>(q.Q);
    const T* KS = static_cast<const T*>(q.K_S);
    qnorm_partial<E, D><<<dim3(nsplit, (unsigned)q.BH), kNormThreads, 0, st>>>(Q, q.m, rows_per_split, part);
    shift_finalize<E, D><<<(unsigned)q.BH, 256, 0, st>>>(part, nsplit, KS, q.rank, q.r, MQ);
    const size_t smem = AttSmem<D>::total;
    cudaError_t e = cudaFuncSetAttribute(attend_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return Status::cuda(e, "attend: smem attribute");
    attend_kernel<E, D><<<dim3((unsigned)ceil_div(q.m, kAttTM), (unsigned)q.BH), kAttThreads, smem, st>>>(
        Q, KS, q.m, q.r, q.rank, q.beta, q.V_S, q.w, q.vmin, q.vmax, MQ, q.O);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend launch");
    return Status::ok();
}

}  // namespace

// Scratch of the CUDA-core attend: query-norm partials and M_Q.
size_t attend_simt_workspace_bytes(int64_t BH, int64_t m) {
    const int nsplit = (int)std::max<int64_t>(1, std::min<int64_t>(64, ceil_div(m, 1024)));
    Carve cv(nullptr, 0);
    cv.take(sizeof(float) * BH * nsplit);
    cv.take(sizeof(float) * BH);
    return cv.used + 256;
}

// Scratch of wildcat_attend: the larger of the CUDA-core scratch and (head
// dims served by the tensor-core kernel) the bf16 copy of V_S^T, the padded w
// and the pivot-key norms.
size_t attend_workspace_bytes(int64_t BH, int64_t m, int d, int r) {
    size_t bytes = attend_simt_workspace_bytes(BH, m);
    if (attend_tc_supported(1, d)) bytes = std::max(bytes, attend_tc_scratch_bytes(BH, d, r) + 256);
    return bytes;
}

Status launch_attend_simt(const AttendRequest& q, cudaStream_t st) {
    const bool bf = q.dtype == 1;
    switch (q.d) {
        case 32: return bf ? run_attend<BF16, 32>(q, st) : run_attend<F32, 32>(q, st);
        case 64: return bf ? run_attend<BF16, 64>(q, st) : run_attend<F32, 64>(q, st);
        case 128: return bf ? run_attend<BF16, 128>(q, st) : run_attend<F32, 128>(q, st);
    }
    return Status::fail(2, "attend: unsupported head dim");
}

// bf16 inputs with d in {64, 128} run on the tensor cores (attend_tc.cu, which
// shifts each query row by |q_i| * max_l |k_S,l| instead of one M_Q per
// instance; both cancel in N / D); everything else on the CUDA-core kernel above.
Status launch_attend(const AttendRequest& q, cudaStream_t st) {
    if (!attend_tc_supported(q.dtype, q.d)) return launch_attend_simt(q, st);
    Carve cv(q.ws, q.ws_bytes);
    void* scratch = cv.take(attend_tc_scratch_bytes(q.BH, q.d, q.r));
    if (!cv.fits()) return Status::fail(4, "attend: workspace too small");
    return launch_attend_tc(q, scratch, st);
}

// ---------------------------------------------------------------------------
// Allocation-free attend (wildcat_attend_noalloc).
//
// Some callers cannot hand the library a workspace: they only hold pointers
// that another component gave them, inside a process whose device memory is
// owned by that component (for example a serving engine that reserves almost
// all of the GPU for its KV cache and routes every allocation through its own
// pool), or they run in a latency-critical loop where a cudaMalloc, which can
// synchronise the device, is not acceptable.  For them the attend's small
// scratch (per-instance query-norm partials and the shift M_Q) lives in the
// fixed device array below instead of a caller workspace.  It runs the
// CUDA-core attend kernel, whose scratch is small enough for a fixed array.
//
// The array is kNoAllocScratchBytes (1 MiB) and exists on every GPU on which
// this library's kernels are loaded, until the process exits.  Host code may
// not pass the array's name to a kernel (on the host it is only a stand-in
// symbol), so the device address is looked up with cudaGetSymbolAddress once
// per device, with that device current, on the first no-alloc call made
// there; make that first call before any stream capture.  The address is
// kept per device ordinal for the life of the process, which assumes the
// device's primary context stays the one in use: after cudaDeviceReset, or
// with another context current on that ordinal, it would be stale.  All calls share
// the array: calls whose kernels overlap on the GPU (for example on two
// streams at once) race on it and must be serialised by the caller.  Every
// scratch word a call reads is written earlier in the same call, so nothing
// needs clearing between calls.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_addr[kNoAllocMaxDevices] = {};

Status attend_scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return Status::cuda(e, "attend_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocMaxDevices) return Status::fail(2, "attend_noalloc: device ordinal above 63");
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess || p == nullptr)
            return Status::cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                                "attend_noalloc: cudaGetSymbolAddress of the static scratch");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return Status::ok();
}
}  // namespace

size_t attend_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

Status launch_attend_noalloc(const AttendRequest& q_in, cudaStream_t st) {
    if (attend_simt_workspace_bytes(q_in.BH, q_in.m) > kNoAllocScratchBytes)
        return Status::fail(2,
                            "wildcat_attend_noalloc: BH and m need more scratch than the 1 MiB static array "
                            "(about 4 * BH * (min(64, ceil(m / 1024)) + 1) bytes); use wildcat_attend with a workspace");
    void* scratch = nullptr;
    const Status s = attend_scratch_address(&scratch);
    if (s.code) return s;
    AttendRequest q = q_in;
    q.ws = scratch;
    q.ws_bytes = kNoAllocScratchBytes;
    return launch_attend_simt(q, st);
}

}  // namespace wildcat
