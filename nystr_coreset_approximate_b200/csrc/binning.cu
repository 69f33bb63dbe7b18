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
// and the optional global pivot indices and per-bin ranks.
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

}  // namespace

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
