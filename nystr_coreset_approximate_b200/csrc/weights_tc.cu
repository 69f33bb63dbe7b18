// weights_tc.cu -- Y = F^T (V, 1_n) on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: W is
// applied to (V, 1_n) before the queries; with the partial Cholesky factor,
// W (V, 1) = F_S^-T Y and Y = F^T (V, 1).  This kernel forms split-K partials
// of Y for bfloat16 values; the back substitution in weights.cu sums them.
//
// One CTA per (128 factor columns, key range, instance); the key range is
// walked in chunks of 64 keys.  Warp roles:
//   warp 0     TMA: the chunk's factor rows F[j0 .. j0+127, keys] (fp32, two
//              128 x 32 boxes, 128-byte swizzle) into a ring of NF stages
//   warp 2     TMA: the chunk's value rows V[keys, 0 .. d) (bf16, MN-major
//              boxes of 64 keys x 64 columns) into stage s of the AB ring
//   warps 4-7  split each factor row into bf16 hi + lo parts, written K-major
//              with the 128-byte swizzle into stage s of the AB ring (thread
//              i converts row i); the factor stage is then released
//   warp 1     one thread issues per chunk two tcgen05.mma groups (hi and lo
//              parts of A, the same B = [V | 1 | 0]) into the fp32
//              accumulator Y (M = 128, N = d + 16) in tensor memory
// The ones column (and zero padding to d + 16) is written once per AB stage.
// Keys past n read as zeros through the tensor maps, so they add nothing.
// The hi/lo split keeps Y accurate to ~2^-17 relative while the factor is
// read from HBM once.  Afterwards warps 4-7 write the CTA's partial Y rows.
// Tiles starting at or past the instance's effective rank do no work (those
// rows of F are zero and the solve never reads them).
//
// Every mbarrier wait is bounded (2 s) and gives up when another role gave
// up; an expiry records WILDCAT_ERR_TIMEOUT in the device status word, the
// CTA drains what it issued (bounded), frees its tensor memory and returns.
// No load uses cluster multicast.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace wildcat {

__device__ int g_weights_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

namespace {

using namespace tc;
constexpr int kWtThreads = 256;
constexpr int kWtKC = 64;  // keys per chunk
constexpr int kWtNF = 3;   // factor staging stages (fp32)
constexpr int kWtNAB = 2;  // converted-operand stages (A hi / lo, B)
constexpr unsigned long long kDrainNs = 100000000ull;

struct WtBars {
    uint64_t f_full[kWtNF], f_empty[kWtNF];
    uint64_t a_full[kWtNAB], b_full[kWtNAB], ab_empty[kWtNAB];
    uint64_t done;
    unsigned tmem_base;
    int abort;
};

template <int D>
struct WtCfg {
    static constexpr int NE = D + 16;                          // value columns + ones column + zero padding
    static constexpr int NBLK = D / 64 + 1;                    // 64-column MN blocks of B (the last holds the ones)
    static constexpr uint32_t f_bytes = 2 * 128 * 128;         // 128 rows x 64 keys fp32: two 128-byte boxes
    static constexpr uint32_t a_bytes = 128 * 128;             // one part: 128 rows x 64 keys bf16
    static constexpr uint32_t b_bytes = NBLK * kWtKC * 128;    // 64 keys x NBLK * 64 columns bf16
    static constexpr uint32_t v_bytes = (D / 64) * kWtKC * 128;  // the V part of B (what the TMA fills)
    static constexpr uint32_t ab_bytes = 2 * a_bytes + b_bytes;
    static constexpr uint32_t off_f = 0;
    static constexpr uint32_t off_ab = off_f + kWtNF * f_bytes;
    static constexpr uint32_t off_bar = off_ab + kWtNAB * ab_bytes;
    static constexpr uint32_t total = off_bar + (uint32_t)sizeof(WtBars);
    static constexpr unsigned tmem_cols = 256;
    static_assert(NE <= 256, "accumulator columns");
    static_assert(total <= 232448, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kWtThreads, 1)
    weights_tc_kernel(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmV,
                      const int32_t* __restrict__ rank, int64_t n, int r, int64_t keys_per_split,
                      float* __restrict__ Ypart, int64_t BH) {
    using C = WtCfg<D>;
    constexpr int NE = C::NE;
    const int b = blockIdx.z;
    const int split = blockIdx.y;
    const int j0 = blockIdx.x * 128;
    if (j0 >= rank[b]) return;  // uniform: the whole CTA leaves before any allocation

    extern __shared__ __align__(1024) unsigned char sm[];
    const unsigned sbase = smem_u32(sm);
    WtBars* bars = reinterpret_cast<WtBars*>(sm + C::off_bar);
    volatile int* abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int64_t l_begin = split * keys_per_split;
    const int64_t l_end = min(n, l_begin + keys_per_split);
    const int nchunks = l_end > l_begin ? (int)ceil_div(l_end - l_begin, kWtKC) : 0;

    if (tid == 0) {
        for (int s = 0; s < kWtNF; ++s) {
            mbar_init(&bars->f_full[s], 1);
            mbar_init(&bars->f_empty[s], 4);  // one arrival per converter warp
        }
        for (int s = 0; s < kWtNAB; ++s) {
            mbar_init(&bars->a_full[s], 4);  // one arrival per converter warp
            mbar_init(&bars->b_full[s], 1);
            mbar_init(&bars->ab_empty[s], 1);
        }
        mbar_init(&bars->done, 1);
        bars->abort = (sbase & 1023u) ? 1 : 0;  // the swizzled layouts need a 1024-byte aligned base
        if (sbase & 1023u) atomicExch(&g_weights_status, 3);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the ones column (value column d) and the zero padding of every AB stage's B
    for (int e = tid; e < kWtNAB * kWtKC; e += kWtThreads) {
        const int s = e / kWtKC, kr = e % kWtKC;
        unsigned char* blk = sm + C::off_ab + s * C::ab_bytes + 2 * C::a_bytes + (D / 64) * (kWtKC * 128);
        const __nv_bfloat16 one = __float2bfloat16_rn(1.f);
        uint4 c0 = make_uint4((uint32_t)(*reinterpret_cast<const uint16_t*>(&one)), 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(blk + swz(kr, 0)) = c0;
        *reinterpret_cast<uint4*>(blk + swz(kr, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
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
    const unsigned tmem = bars->tmem_base;
    const bool go = *abort_flag == 0;
    auto give_up = [&]() {
        *abort_flag = 1;
        atomicExch(&g_weights_status, 5);
    };

    if (warp == 0) {
        // ---------------------------------------------------- factor rows (TMA)
        if (lane == 0 && go) {
            prefetch_tmap(&tmF);
            int c = 0;
            bool ok = true;
            for (; c < nchunks; ++c) {
                const int s = c % kWtNF;
                if (c >= kWtNF &&
                    !(ok = mbar_wait_suspend(&bars->f_empty[s], (unsigned)((c / kWtNF) - 1) & 1u, abort_flag)))
                    break;
                mbar_expect_tx(&bars->f_full[s], C::f_bytes);
                const int x = (int)(l_begin + (int64_t)c * kWtKC);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    tma_load_3d(sbase + C::off_f + s * C::f_bytes + h * (128 * 128), &tmF, x + 32 * h, j0, b,
                                &bars->f_full[s]);
            }
            if (!ok) give_up();
            if (*abort_flag)
                for (int k = std::max(0, c - kWtNF); k < c; ++k)
                    mbar_wait(&bars->f_full[k % kWtNF], (unsigned)(k / kWtNF) & 1u, kDrainNs);
        }
    } else if (warp == 2) {
        // ----------------------------------------------------- value rows (TMA)
        if (lane == 0 && go) {
            prefetch_tmap(&tmV);
            int c = 0;
            bool ok = true;
            for (; c < nchunks; ++c) {
                const int s = c % kWtNAB;
                if (c >= kWtNAB &&
                    !(ok = mbar_wait_suspend(&bars->ab_empty[s], (unsigned)((c / kWtNAB) - 1) & 1u, abort_flag)))
                    break;
                mbar_expect_tx(&bars->b_full[s], C::v_bytes);
                const int y = (int)(l_begin + (int64_t)c * kWtKC);
#pragma unroll
                for (int blk = 0; blk < D / 64; ++blk)
                    tma_load_3d(sbase + C::off_ab + s * C::ab_bytes + 2 * C::a_bytes + blk * (kWtKC * 128), &tmV,
                                64 * blk, y, b, &bars->b_full[s]);
            }
            if (!ok) give_up();
            if (*abort_flag)
                for (int k = std::max(0, c - kWtNAB); k < c; ++k)
                    mbar_wait(&bars->b_full[k % kWtNAB], (unsigned)(k / kWtNAB) & 1u, kDrainNs);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- tensor cores
        if (lane == 0 && go) {
            constexpr uint32_t idesc = idesc_bf16_bmn(128, NE);
            bool ok = true;
            int c = 0;
            for (; c < nchunks; ++c) {
                const int s = c % kWtNAB;
                const unsigned ph = (unsigned)(c / kWtNAB) & 1u;
                if (!(ok = mbar_wait_suspend(&bars->a_full[s], ph, abort_flag) &&
                           mbar_wait_suspend(&bars->b_full[s], ph, abort_flag)))
                    break;
                tc_fence_after();
                const unsigned st = sbase + C::off_ab + s * C::ab_bytes;
                const unsigned sB = st + 2 * C::a_bytes;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int kk = 0; kk < kWtKC / 16; ++kk)
                        mma_bf16(tmem, umma_desc(st + part * C::a_bytes + kk * 32),
                                 umma_desc_mn(sB + kk * 16 * 128, kWtKC * 128), idesc, (c > 0 || part > 0 || kk > 0) ? 1 : 0);
                }
                mma_commit(&bars->ab_empty[s]);
            }
            if (!ok) give_up();
            mma_commit(&bars->done);  // every product issued has finished when this arrives
            mbar_wait(&bars->done, 0, ok ? kWaitLimitNs : kDrainNs);
        }
    } else if (warp >= 4) {
        // ------------------------------------------- hi / lo split, then Y out
        const int row = tid - 128;  // factor column j0 + row = TMEM lane
        bool ok = go;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int sf = c % kWtNF, sa = c % kWtNAB;
            const bool got = mbar_wait_suspend(&bars->f_full[sf], (unsigned)(c / kWtNF) & 1u, abort_flag) &&
                             (c < kWtNAB ||
                              mbar_wait_suspend(&bars->ab_empty[sa], (unsigned)((c / kWtNAB) - 1) & 1u, abort_flag));
            ok = __all_sync(0xffffffffu, got);
            if (!ok) break;
            const unsigned char* frow = sm + C::off_f + sf * C::f_bytes + row * 128;
            unsigned char* ahi = sm + C::off_ab + sa * C::ab_bytes + row * 128;
            unsigned char* alo = ahi + C::a_bytes;
#pragma unroll
            for (int k = 0; k < 8; ++k) {  // 8 keys per 16-byte piece of the bf16 row
                const unsigned char* fb = frow + (k >> 2) * (128 * 128);
                const int c0 = (2 * k) & 7;  // first fp32 piece (4 keys) of this group in its box
                const float4 x0 = *reinterpret_cast<const float4*>(fb + ((c0 ^ (row & 7)) << 4));
                const float4 x1 = *reinterpret_cast<const float4*>(fb + (((c0 + 1) ^ (row & 7)) << 4));
                const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(xs[2 * e], xs[2 * e + 1]);
                    const float2 hf = __bfloat1622float2(h);
                    const __nv_bfloat162 g = __floats2bfloat162_rn(xs[2 * e] - hf.x, xs[2 * e + 1] - hf.y);
                    hi[e] = *reinterpret_cast<const uint32_t*>(&h);
                    lo[e] = *reinterpret_cast<const uint32_t*>(&g);
                }
                const unsigned off = (unsigned)((k ^ (row & 7)) << 4);
                *reinterpret_cast<uint4*>(ahi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(alo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            fence_async_smem();  // the generic-proxy writes become visible to the tensor cores
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->f_empty[sf]);
                mbar_arrive(&bars->a_full[sa]);
            }
        }
        if (!ok && lane == 0) give_up();
        // -- the CTA's partial Y rows (factor columns j0 + row) --
        if (ok && nchunks > 0) ok = __all_sync(0xffffffffu, mbar_wait_suspend(&bars->done, 0, abort_flag));
        const int je = j0 + row;
        if (ok) {
            tc_fence_after();
            float* y = Ypart + (((int64_t)split * BH + b) * r + je) * (D + 1);
#pragma unroll 1
            for (int c0 = 0; c0 < NE; c0 += 16) {
                float vv[16];
                if (nchunks > 0) {
                    tmem_ld16(tmem + ((unsigned)(32 * (warp & 3)) << 16) + c0, vv);
                } else {
#pragma unroll
                    for (int k = 0; k < 16; ++k) vv[k] = 0.f;
                }
                if (je < r) {
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        if (c0 + k <= D) y[c0 + k] = vv[k];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::tmem_cols) : "memory");
    }
}

template <int D>
Status run_wt(const float* F, const void* V, const int32_t* rank, int64_t BH, int64_t n, int r, int nsplit,
              int64_t keys_per_split, float* Ypart, cudaStream_t st) {
    using C = WtCfg<D>;
    CUtensorMap tmF, tmV;
    const bool ok =
        make_tmap_3d(&tmF, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, F, (uint64_t)n, (uint64_t)r, (uint64_t)BH, n * 4ull,
                     (uint64_t)r * n * 4ull, 32, 128) &&
        make_tmap_3d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, V, D, (uint64_t)n, (uint64_t)BH, D * 2ull,
                     (uint64_t)n * D * 2ull, 64, kWtKC);
    if (!ok) return Status::fail(3, "weights_tc: tensor map encoding failed");
    cudaError_t e = cudaFuncSetAttribute(weights_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::total);
    if (e != cudaSuccess) return Status::cuda(e, "weights_tc: smem attribute");
    weights_tc_kernel<D><<<dim3((unsigned)ceil_div(r, 128), nsplit, (unsigned)BH), kWtThreads, C::total, st>>>(
        tmF, tmV, rank, n, r, keys_per_split, Ypart, BH);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "weights_tc launch");
    return Status::ok();
}

}  // namespace

// bf16 values, d in {64, 128}, and n % 4 == 0 (16-byte aligned factor rows).
bool weights_tc_supported(int dtype, int d, int64_t n) { return dtype == 1 && (d == 64 || d == 128) && n % 4 == 0; }

// Key splits of the tensor-core kernel.  One CTA runs per SM at a time, so
// the time is about (waves of CTAs) x (chunks per CTA); each split also
// writes, and the solve reads back, one partial Y of every column tile.  The
// split count minimising the sum (in units of one chunk's HBM traffic per SM)
// is taken, keeping at least 8 chunks of 64 keys per CTA.
int64_t weights_tc_keys_per_split(int64_t BH, int64_t n, int d, int r, int sms) {
    const int64_t tiles = ceil_div(r, 128) * BH;
    const int64_t chunks = ceil_div(n, kWtKC);
    const double chunk_bytes = 128.0 * kWtKC * 4 + (double)kWtKC * d * 2;  // F and V per chunk
    const double y_per_split = (double)tiles * 128 * (d + 1) * 4 * 2 / sms / chunk_bytes;
    int64_t best_ns = 1;
    double best = -1.0;
    for (int64_t ns = 1; ns <= 512 && ns <= chunks; ++ns) {
        const int64_t cpc = ceil_div(chunks, ns);
        if (ns > 1 && cpc < 8) break;
        const double t = (double)ceil_div(tiles * ns, sms) * cpc + ns * y_per_split;
        if (best < 0 || t < best) {
            best = t;
            best_ns = ns;
        }
    }
    return ceil_div(chunks, best_ns) * kWtKC;
}

Status launch_weights_tc(const float* F, const void* V, const int32_t* rank, int64_t BH, int64_t n, int d, int r,
                         int nsplit, int64_t keys_per_split, float* Ypart, cudaStream_t st) {
    if ((reinterpret_cast<uintptr_t>(F) & 15u) || (reinterpret_cast<uintptr_t>(V) & 15u))
        return Status::fail(1, "weights_tc: F and V must be 16-byte aligned");
    switch (d) {
        case 64: return run_wt<64>(F, V, rank, BH, n, r, nsplit, keys_per_split, Ypart, st);
        case 128: return run_wt<128>(F, V, rank, BH, n, r, nsplit, keys_per_split, Ypart, st);
    }
    return Status::fail(2, "weights_tc: unsupported head dim");
}

int read_weights_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_weights_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_weights_status, &z, sizeof(int));
    }
    return v;
}

}  // namespace wildcat
