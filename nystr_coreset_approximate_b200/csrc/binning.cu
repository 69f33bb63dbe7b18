// binning.cu -- divide-and-conquer glue for the binned WildCat forward.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: to use the
// GPU's parallelism the n keys of an instance are cut into B bins, each
// with its own coreset of r / B pivots.  With contiguous equal bins, bin q of
// instance b is simply instance b * B + q of the [BH * B, n / B, d] view of
// K and V, so the select and weights kernels run unchanged on that view; the
// union coreset is the [BH, r, d] view of their outputs.  This kernel does
// the remaining glue: the value range over all n keys (the minimum and
// maximum of the per-bin ranges), the attend's row count (all r union rows;
// rows past a bin's rank are zero in K_S, V_S and w and contribute nothing),
// and the optional global pivot indices and per-bin ranks.  It also holds the
// per-instance key mean used for recentring (Sec. 2: softmax attention is
// invariant under a global shift of the keys).
#include "common.cuh"
#include "internal.h"

namespace wildcat {

namespace {

__global__ void binning_finish_kernel(const float* vmin_b, const float* vmax_b, const int32_t* S_b,
                                      const int32_t* rank_b, int64_t BH, int nbins, int64_t nb, int rb, int d,
                                      float* vmin, float* vmax, int32_t* rank_att, int32_t* S_out,
                                      int32_t* rank_out) {
    const int64_t b = blockIdx.x;
    const int r = rb * nbins;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float lo = INFINITY, hi = -INFINITY;
        for (int q = 0; q < nbins; ++q) {
            lo = fminf(lo, vmin_b[(b * nbins + q) * d + c]);
            hi = fmaxf(hi, vmax_b[(b * nbins + q) * d + c]);
        }
        vmin[b * d + c] = lo;
        vmax[b * d + c] = hi;
    }
    if (threadIdx.x == 0) rank_att[b] = r;
    if (S_out)
        for (int e = threadIdx.x; e < r; e += blockDim.x) {
            const int q = e / rb;
            const int32_t s = S_b[b * r + e];
            S_out[b * r + e] = s >= 0 ? (int32_t)(q * nb + s) : -1;
        }
    if (rank_out)
        for (int q = threadIdx.x; q < nbins; q += blockDim.x) rank_out[b * nbins + q] = rank_b[b * nbins + q];
}

constexpr int kMeanThreads = 256;

template <typename E>
__global__ void __launch_bounds__(kMeanThreads) key_mean_partial(const typename E::T* K, int64_t n, int d,
                                                                 int64_t rows_per_split, double* part) {
    // part [BH, nsplit, d]: fp64 column sums of a slice of the keys
    const int64_t b = blockIdx.y;
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int slots = kMeanThreads / d;
    const int c = threadIdx.x % d, slot = threadIdx.x / d;
    const int64_t l0 = split * rows_per_split, l1 = min(n, l0 + rows_per_split);
    double acc = 0.0;
    if (slot < slots)
        for (int64_t l = l0 + slot; l < l1; l += slots) acc += (double)E::to_float(K[(b * n + l) * d + c]);
    __shared__ double red[kMeanThreads];
    red[threadIdx.x] = acc;
    __syncthreads();
    if (slot == 0) {
        for (int k = 1; k < slots; ++k) acc += red[k * d + c];
        part[(b * nsplit + split) * d + c] = acc;
    }
}

__global__ void key_mean_finalize(const double* part, int nsplit, int64_t BH, int64_t n, int d, float* kbar) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= BH * d) return;
    const int64_t b = t / d;
    const int c = (int)(t % d);
    double s = 0.0;
    for (int k = 0; k < nsplit; ++k) s += part[(b * nsplit + k) * d + c];
    kbar[t] = (float)(s / (double)n);
}

int mean_splits(int64_t BH, int64_t n) {
    int64_t s = ceil_div(296, BH > 0 ? BH : 1);
    s = s < 1 ? 1 : (s > 64 ? 64 : s);
    const int64_t cap = n / 256 > 0 ? n / 256 : 1;
    return (int)(s < cap ? s : cap);
}

}  // namespace

size_t key_mean_workspace_bytes(int64_t BH, int64_t n, int d) {
    return sizeof(double) * (size_t)BH * mean_splits(BH, n) * d + 256;
}

Status launch_key_mean(const void* K, int dtype, int64_t BH, int64_t n, int d, void* ws, float* kbar,
                       cudaStream_t st) {
    const int nsplit = mean_splits(BH, n);
    const int64_t rows = ceil_div(n, nsplit);
    double* part = static_cast<double*>(ws);
    if (dtype == 1)
        key_mean_partial<BF16><<<dim3(nsplit, (unsigned)BH), kMeanThreads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(K), n, d, rows, part);
    else
        key_mean_partial<F32><<<dim3(nsplit, (unsigned)BH), kMeanThreads, 0, st>>>(static_cast<const float*>(K), n,
                                                                                   d, rows, part);
    key_mean_finalize<<<(unsigned)ceil_div(BH * d, 256), 256, 0, st>>>(part, nsplit, BH, n, d, kbar);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "key mean launch");
    return Status::ok();
}

Status launch_binning_finish(const float* vmin_b, const float* vmax_b, const int32_t* S_b, const int32_t* rank_b,
                             int64_t BH, int nbins, int64_t nb, int rb, int d, float* vmin, float* vmax,
                             int32_t* rank_att, int32_t* S_out, int32_t* rank_out, cudaStream_t st) {
    binning_finish_kernel<<<(unsigned)BH, 128, 0, st>>>(vmin_b, vmax_b, S_b, rank_b, BH, nbins, nb, rb, d, vmin, vmax,
                                                         rank_att, S_out, rank_out);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "binning finish launch");
    return Status::ok();
}

}  // namespace wildcat
