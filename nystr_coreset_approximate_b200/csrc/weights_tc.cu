// weights_tc.cu -- Y = F^T (V, 1_n) on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2: W is
// applied to (V, 1_n) before the queries; with the partial Cholesky factor,
// W (V, 1) = F_S^-T Y and Y = F^T (V, 1).  This kernel forms split-K partials
// of Y for bfloat16 values; the back substitution in weights.cu sums them.
//
// One CTA (256 threads) per (128 factor columns, key slice, instance).  Per
// chunk of 64 keys:
//   A = F[j0 .. j0+127, keys] (fp32 in HBM) split into bf16 hi + lo parts,
//       written K-major with 128-byte swizzling;
//   B = [V | 1 | 0] for the same keys (d + 16 columns, bf16), MN-major: V's
//       rows are copied as they are, the ones column and the zero padding
//       are written in shared memory;
//   two tcgen05.mma (hi and lo) per 16 keys accumulate Y in tensor memory
//   (M = 128, N = d + 16, fp32).
// The epilogue writes the partial Y rows of the CTA's factor columns.
// Tiles starting at or past the instance's effective rank do no work (those
// rows of F are zero and the solve never reads them).
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace wildcat {

__device__ int g_weights_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

namespace {

using namespace tc;
constexpr int kWtThreads = 256;
constexpr int kWtKC = 64;  // keys per chunk

template <int D>
struct WtSmem {
    static constexpr int NE = D + 16;
    static constexpr int NB = (NE + 63) / 64;                          // 64-column MN blocks of B
    static constexpr size_t ahi = 0;                                   // 128 x 64 bf16
    static constexpr size_t alo = ahi + 128 * 128;
    static constexpr size_t b = alo + 128 * 128;                       // NB blocks of 64 keys x 128 B
    static constexpr size_t stage = b + (size_t)NB * kWtKC * 128;      // one pipeline stage
    static constexpr size_t bar = 2 * stage;                           // two stages, then the barriers
    static constexpr size_t total = bar + 64 + 1024;
    static constexpr unsigned tmem_cols = 256;
};

template <int D>
__global__ void __launch_bounds__(kWtThreads)
    weights_tc_kernel(const float* __restrict__ F, const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ rank,
                      int64_t n, int r, int64_t keys_per_split, float* __restrict__ Ypart, int64_t BH) {
    using L = WtSmem<D>;
    constexpr int NE = L::NE;
    const int64_t b = blockIdx.z;
    const int split = blockIdx.y;
    const int j0 = blockIdx.x * 128;
    if (j0 >= rank[b]) return;  // uniform: the whole CTA leaves before any allocation

    extern __shared__ unsigned char sm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + L::bar);  // one per stage
    unsigned* tmem_slot = reinterpret_cast<unsigned*>(sm + L::bar + 16);
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(L::tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = *tmem_slot;
    constexpr uint32_t idesc = idesc_bf16_bmn(128, NE);

    const int64_t l_begin = split * keys_per_split;
    const int64_t l_end = min(n, l_begin + keys_per_split);
    const int nchunks = l_end > l_begin ? (int)ceil_div(l_end - l_begin, kWtKC) : 0;
    const float* Fb = F + b * (int64_t)r * n;
    const __nv_bfloat16* Vb = V + b * n * D;
    const int row = tid >> 1, half = tid & 1;  // A: factor row j0 + row, 32 keys from half * 32
    const int j = j0 + row;

    // F rows of chunk c into registers (global loads left in flight)
    auto load_a = [&](int c, float (&v)[32]) {
        const int64_t l0 = l_begin + (int64_t)c * kWtKC;
        const float* src = Fb + (int64_t)j * n + l0 + half * 32;
        const bool full = j < r && l0 + half * 32 + 32 <= l_end;
        if (full) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 x = __ldcs(reinterpret_cast<const float4*>(src) + k);
                v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int64_t l = l0 + half * 32 + k;
                v[k] = (j < r && l < l_end) ? __ldcs(Fb + (int64_t)j * n + l) : 0.f;
            }
        }
    };
    // B of chunk c into stage st: V rows (MN-major: key = row, 64 value
    // columns per 128-byte row) by cp.async, then the ones column and zeros
    auto load_b = [&](int c, int st) {
        const int64_t l0 = l_begin + (int64_t)c * kWtKC;
        unsigned char* sb = sm + st * L::stage + L::b;
        const unsigned sB = smem_u32(sb);
        for (int e = tid; e < kWtKC * (D / 8); e += kWtThreads) {
            const int kr = e / (D / 8), c8 = e % (D / 8);  // key row, 16-byte chunk along d
            const int64_t l = l0 + kr;
            const bool okl = l < l_end;
            const unsigned dst = (c8 >> 3) * (kWtKC * 128) + swz(kr, c8 & 7);
            cp_async16_zfill(sB + dst, Vb + (okl ? l : l0) * D + c8 * 8, okl);
        }
        cp_async_commit();
        for (int kr = tid; kr < kWtKC; kr += kWtThreads) {
            const bool okl = l0 + kr < l_end;
            const int mb = D / 64;  // block holding columns D .. D + 15 (chunks 0 and 1)
            const __nv_bfloat16 one = __float2bfloat16_rn(okl ? 1.f : 0.f);
            uint4 c0 = make_uint4(0u, 0u, 0u, 0u);
            c0.x = (uint32_t)(*reinterpret_cast<const uint16_t*>(&one));
            *reinterpret_cast<uint4*>(sb + mb * (kWtKC * 128) + swz(kr, 0)) = c0;
            *reinterpret_cast<uint4*>(sb + mb * (kWtKC * 128) + swz(kr, 1)) = make_uint4(0u, 0u, 0u, 0u);
        }
    };

    // Two stages: while the tensor cores work on chunk c, the V rows of chunk
    // c + 1 land by cp.async and the F rows of chunks c + 1 and c + 2 are in
    // flight into registers (two register sets, the loop unrolled by two).
    // Stage s is rewritten only after the MMA that read it (chunk c - 1 for
    // B, chunk c - 2 for A) has committed on mbar[s].
    bool ok = true;
    int issued = 0;  // MMA commits so far (commit k arrives on mbar[k & 1], phase k >> 1)
    auto step = [&](int c, float (&v)[32]) -> bool {
        const int st = c & 1;
        if (c >= 1) {
            // chunk c - 1's MMA has read stage st ^ 1: free it for chunk c + 1
            const bool w = mbar_wait(&mbar[(c - 1) & 1], ((c - 1) >> 1) & 1);
            if (__syncthreads_or(!w)) return false;
            tc_fence_after();
        }
        if (c + 1 < nchunks) load_b(c + 1, st ^ 1);
        // A of chunk c: bf16 hi / lo, K-major, 128-byte swizzle
        unsigned char* sa = sm + st * L::stage;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = v[8 * q + 2 * e], a1 = v[8 * q + 2 * e + 1];
                const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                const float2 hf = __bfloat1622float2(h);
                const __nv_bfloat162 g = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                hi[e] = *reinterpret_cast<const uint32_t*>(&h);
                lo[e] = *reinterpret_cast<const uint32_t*>(&g);
            }
            const unsigned off = swz(row, half * 4 + q);
            *reinterpret_cast<uint4*>(sa + L::ahi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sa + L::alo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        if (c + 2 < nchunks) load_a(c + 2, v);
        if (c + 1 < nchunks)
            cp_async_wait_group<1>();  // chunk c's V rows (chunk c + 1's may still fly)
        else
            cp_async_wait_all();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const unsigned sAhi = smem_u32(sa + L::ahi), sAlo = smem_u32(sa + L::alo), sB = smem_u32(sa + L::b);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const unsigned sap = part ? sAlo : sAhi;
#pragma unroll
                for (int kk = 0; kk < kWtKC / 16; ++kk)
                    mma_bf16(tmem, umma_desc(sap + kk * 32), umma_desc_mn(sB + kk * 16 * 128, kWtKC * 128), idesc,
                             (c > 0 || part > 0 || kk > 0) ? 1 : 0);
            }
            mma_commit(&mbar[st]);
        }
        ++issued;
        return true;
    };
    float v0[32], v1[32];
    if (nchunks > 0) {
        load_b(0, 0);
        load_a(0, v0);
        if (nchunks > 1) load_a(1, v1);
    }
    for (int c = 0; c < nchunks; c += 2) {
        if (!step(c, v0)) { ok = false; break; }
        if (c + 1 < nchunks && !step(c + 1, v1)) { ok = false; break; }
    }
    // the last commit covers every MMA issued before it
    if (issued > 0) {
        const int k = issued - 1;
        const bool w = mbar_wait(&mbar[k & 1], (k >> 1) & 1);
        if (__syncthreads_or(!w)) ok = false;
        tc_fence_after();
    }
    // -- epilogue: warps 0-3 read their 32 TMEM lanes (= factor columns j0 + lane row) --
    if (ok && warp < 4 && issued > 0) {
        const int rowe = warp * 32 + (tid & 31);
        const int je = j0 + rowe;
        float* y = Ypart + (((int64_t)split * BH + b) * r + je) * (D + 1);
#pragma unroll 1
        for (int c0 = 0; c0 < D + 16; c0 += 16) {
            float vv[16];
            tmem_ld16(tmem + ((unsigned)(warp * 32) << 16) + c0, vv);
            if (je < r) {
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (c0 + k <= D) y[c0 + k] = vv[k];
            }
        }
    } else if (ok && warp < 4 && issued == 0) {
        const int je = j0 + warp * 32 + (tid & 31);
        if (je < r) {
            float* y = Ypart + (((int64_t)split * BH + b) * r + je) * (D + 1);
            for (int c = 0; c <= D; ++c) y[c] = 0.f;
        }
    }
    if (!ok) {
        if (tid == 0) atomicExch(&g_weights_status, 5);
        // bounded wait for the last MMA still in flight before its memory is freed
        if (issued > 0) mbar_wait(&mbar[(issued - 1) & 1], ((issued - 1) >> 1) & 1);
        cp_async_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::tmem_cols) : "memory");
    }
}

template <int D>
Status run_wt(const float* F, const void* V, const int32_t* rank, int64_t BH, int64_t n, int r, int nsplit,
              int64_t keys_per_split, float* Ypart, cudaStream_t st) {
    using L = WtSmem<D>;
    cudaError_t e = cudaFuncSetAttribute(weights_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::total);
    if (e != cudaSuccess) return Status::cuda(e, "weights_tc: smem attribute");
    weights_tc_kernel<D><<<dim3((unsigned)ceil_div(r, 128), nsplit, (unsigned)BH), kWtThreads, L::total, st>>>(
        F, static_cast<const __nv_bfloat16*>(V), rank, n, r, keys_per_split, Ypart, BH);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "weights_tc launch");
    return Status::ok();
}

}  // namespace

// bf16 values, d in {64, 128}, and n % 4 == 0 (16-byte aligned factor rows).
bool weights_tc_supported(int dtype, int d, int64_t n) { return dtype == 1 && (d == 64 || d == 128) && n % 4 == 0; }

Status launch_weights_tc(const float* F, const void* V, const int32_t* rank, int64_t BH, int64_t n, int d, int r,
                         int nsplit, int64_t keys_per_split, float* Ypart, cudaStream_t st) {
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
