// attend_tc.cu -- weighted-coreset attention on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2 plug-in
// estimator and Alg. 3 WtdAttn, for bfloat16 inputs:
//     P = exp(beta Q K_S^T - beta M_Q),   N = P [V_S | w],   O = clip(N_v / N_w).
//
// One CTA (128 threads) per tile of 128 queries of one instance.  Per chunk
// of 128 coreset rows:
//   GEMM1  S = Q K_S^T     tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//                          M = 128, N = 128, K = d
//   exp    thread i (= TMEM lane i = query row i) loads its row of S with
//          tcgen05.ld, forms P = exp(beta s - beta M_Q) and writes it as
//          bf16 into shared memory in the UMMA K-major 128-byte-swizzled
//          layout
//   GEMM2  N += P [V_S | w]  with [V_S | w] split as hi + lo bf16 parts (two
//          MMAs), M = 128, N = d + 16, K = 128, accumulated in TMEM across
//          chunks.  The numerator and the denominator use the same rounded P.
// Epilogue: thread i reads its row of N and writes O_i = clip(N_i / N_iw).
//
// Operands are staged with cp.async into the swizzled layout (16-byte
// chunk c of row r of an 8-row, 128-byte-wide atom sits at chunk c ^ (r % 8)).
// Every mbarrier wait is bounded by a time limit; on expiry the kernel sets
// the device status word, stops issuing work, frees its TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace wildcat {

__device__ int g_device_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

namespace {

using namespace tc;
constexpr int kTcThreads = 128;
unsigned long long g_force_timeout_ns = 0;  // test hook, 0 = off
constexpr int kTcRC = 128;  // coreset rows per chunk

template <int D>
struct TcSmem {
    static constexpr int NE = D + 16;                         // value columns + w + zero padding
    static constexpr int KB1 = D / 64;                        // 128-byte K blocks of Q / K_S rows
    static constexpr int KB2 = kTcRC / 64;                    // 128-byte K blocks of P / [V_S|w]^T rows
    static constexpr size_t a1 = 0;                           // Q tile    128 x D
    static constexpr size_t b1 = a1 + (size_t)KB1 * 128 * 128;  // K_S chunk 128 x D
    static constexpr size_t a2 = b1 + (size_t)KB1 * 128 * 128;  // P         128 x 128
    static constexpr size_t b2h = a2 + (size_t)KB2 * 128 * 128; // [V_S|w]^T hi  NE x 128
    static constexpr size_t b2l = b2h + (size_t)KB2 * NE * 128;
    static constexpr size_t bar = b2l + (size_t)KB2 * NE * 128;  // 2 mbarriers + TMEM base
    static constexpr size_t total = bar + 64 + 1024;            // + slack for 1024-byte alignment
    static constexpr unsigned tmem_cols = (128 + NE) <= 256 ? 256u : 512u;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    attend_tc_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K_S,
                     const __nv_bfloat16* __restrict__ B2h, const __nv_bfloat16* __restrict__ B2l, int64_t m, int r,
                     int rpad, const int32_t* __restrict__ rank, float beta, const float* __restrict__ vmin,
                     const float* __restrict__ vmax, const float* __restrict__ MQ, float* __restrict__ O,
                     unsigned long long force_timeout_ns) {
    using L = TcSmem<D>;
    constexpr int NE = L::NE;
    extern __shared__ unsigned char sm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const unsigned sA1 = smem_u32(sm + L::a1), sB1 = smem_u32(sm + L::b1), sA2 = smem_u32(sm + L::a2);
    const unsigned sB2h = smem_u32(sm + L::b2h), sB2l = smem_u32(sm + L::b2l);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + L::bar);
    unsigned* tmem_base_slot = reinterpret_cast<unsigned*>(sm + L::bar + 16);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t b = blockIdx.y;
    const int64_t i0 = (int64_t)blockIdx.x * 128;
    const int rr = rank[b];
    const float shift = beta * MQ[b];

    if (tid == 0) {
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_slot)),
                     "r"(L::tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Q tile: row tid, D/8 chunks of 16 bytes
    {
        const int64_t i = i0 + tid;
        const bool ok = i < m;
        const __nv_bfloat16* src = Q + ((b * m + (ok ? i : 0)) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
            cp_async16_zfill(sA1 + (c >> 3) * (128 * 128) + swz(tid, c & 7), src + c * 8, ok);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = *tmem_base_slot;
    const unsigned tmem_S = tmem, tmem_N = tmem + 128;
    const unsigned lane_off = (unsigned)(warp * 32) << 16;
    constexpr uint32_t id1 = idesc_bf16(128, kTcRC), id2 = idesc_bf16(128, NE);

    bool ok = true;
    int chunk = 0;
    if (force_timeout_ns) {
        // test hook: wait for a barrier phase that nothing will complete
        const bool w = mbar_wait(&mbar[1], 0, force_timeout_ns);
        if (__syncthreads_or(!w)) ok = false;
    }
    for (int l0 = 0; ok && l0 < rr; l0 += kTcRC, ++chunk) {
        // -- stage K_S chunk (row tid) and the hi/lo [V_S|w]^T chunk --
        {
            const int l = l0 + tid;
            const bool okr = l < rr;
            const __nv_bfloat16* src = K_S + ((b * r + (okr ? l : 0)) * (int64_t)D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                cp_async16_zfill(sB1 + (c >> 3) * (128 * 128) + swz(tid, c & 7), src + c * 8, okr);
            for (int e = tid; e < NE * (kTcRC / 8); e += kTcThreads) {
                const int row = e / (kTcRC / 8), c = e % (kTcRC / 8);
                const int64_t off = ((b * NE + row) * (int64_t)rpad) + l0 + c * 8;
                const unsigned dst = (c >> 3) * (NE * 128) + swz(row, c & 7);
                cp_async16_zfill(sB2h + dst, B2h + off, true);
                cp_async16_zfill(sB2l + dst, B2l + off, true);
            }
            cp_async_wait_all();
            fence_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // -- GEMM1: S = Q K_S^T --
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const unsigned off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                mma_bf16(tmem_S, umma_desc(sA1 + off), umma_desc(sB1 + off), id1, kk > 0);
            }
            mma_commit(&mbar[0]);
        }
        const bool w1 = mbar_wait(&mbar[0], chunk & 1);
        if (__syncthreads_or(!w1)) { ok = false; break; }
        tc_fence_after();
        // -- P = exp(beta s - beta M_Q) in bf16, written as the K-major A operand of GEMM2 --
#pragma unroll 1
        for (int c0 = 0; c0 < kTcRC; c0 += 16) {
            float v[16];
            tmem_ld16(tmem_S + lane_off + c0, v);
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int l = l0 + c0 + 2 * k;
                const float p0 = l < rr ? expf(beta * v[2 * k] - shift) : 0.f;
                const float p1 = l + 1 < rr ? expf(beta * v[2 * k + 1] - shift) : 0.f;
                const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                pk[k] = *reinterpret_cast<const uint32_t*>(&h);
            }
            const int cc = c0 >> 3;  // 16-byte chunk index along the 128 coreset columns
            unsigned char* base = sm + L::a2 + (cc >> 3) * (128 * 128);
            *reinterpret_cast<uint4*>(base + swz(tid, cc & 7)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(base + swz(tid, (cc + 1) & 7)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // -- GEMM2: N += P [V_S|w] (hi and lo parts) --
        if (tid == 0) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const unsigned sb = part ? sB2l : sB2h;
#pragma unroll
                for (int kk = 0; kk < kTcRC / 16; ++kk) {
                    const unsigned offa = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                    const unsigned offb = (kk >> 2) * (NE * 128) + (kk & 3) * 32;
                    mma_bf16(tmem_N, umma_desc(sA2 + offa), umma_desc(sb + offb), id2,
                             (chunk > 0 || part > 0 || kk > 0) ? 1 : 0);
                }
            }
            mma_commit(&mbar[1]);
        }
        const bool w2 = mbar_wait(&mbar[1], chunk & 1);
        if (__syncthreads_or(!w2)) { ok = false; break; }
        tc_fence_after();
    }

    cp_async_wait_all();  // the Q tile when the loop did not run
    // -- epilogue: O = clip(N_v / N_w).  tcgen05.ld is warp-collective, so
    //    every lane loads; only the stores depend on the row being < m. --
    const int64_t i = i0 + tid;
    const bool row_ok = i < m;
    if (ok) {
        float* o = O + (b * m + (row_ok ? i : 0)) * D;
        const float* lo = vmin + b * D;
        const float* hi = vmax + b * D;
        if (rr == 0) {
            if (row_ok)
                for (int c = 0; c < D; ++c) o[c] = lo[c];  // 0 / 0 clipped to v_min
        } else {
            float wv[16];
            tmem_ld16(tmem_N + lane_off + D, wv);
            const float den = wv[0];
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float v[16];
                tmem_ld16(tmem_N + lane_off + c0, v);
                if (row_ok) {
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        float4 out;
                        out.x = fminf(fmaxf(v[k] / den, lo[c0 + k]), hi[c0 + k]);
                        out.y = fminf(fmaxf(v[k + 1] / den, lo[c0 + k + 1]), hi[c0 + k + 1]);
                        out.z = fminf(fmaxf(v[k + 2] / den, lo[c0 + k + 2]), hi[c0 + k + 2]);
                        out.w = fminf(fmaxf(v[k + 3] / den, lo[c0 + k + 3]), hi[c0 + k + 3]);
                        *reinterpret_cast<float4*>(o + c0 + k) = out;
                    }
                }
            }
        }
    } else if (tid == 0) {
        atomicExch(&g_device_status, 5);
    }
    if (!ok && chunk > 0) {
        // give outstanding tensor-core work one more bounded chance to retire
        mbar_wait(&mbar[0], chunk & 1);
        mbar_wait(&mbar[1], chunk & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::tmem_cols) : "memory");
    }
}

// [V_S | w | 0]^T split into bf16 hi and lo parts: B2[b, c, l] for c < D + 16, l < rpad.
template <int D>
__global__ void b2_prep_kernel(const float* __restrict__ V_S, const float* __restrict__ w, const int32_t* rank, int r,
                               int rpad, __nv_bfloat16* __restrict__ B2h, __nv_bfloat16* __restrict__ B2l) {
    constexpr int NE = D + 16;
    const int64_t b = blockIdx.z;
    const int c = blockIdx.y;
    const int l = blockIdx.x * blockDim.x + threadIdx.x;
    if (l >= rpad) return;
    const int rr = rank[b];
    float v = 0.f;
    if (l < rr) v = c < D ? V_S[(b * r + l) * (int64_t)D + c] : (c == D ? w[b * r + l] : 0.f);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(h));
    const int64_t at = (b * NE + c) * (int64_t)rpad + l;
    B2h[at] = h;
    B2l[at] = lo;
}

template <int D>
Status run_tc(const AttendRequest& q, const float* MQ, void* b2ws, cudaStream_t st) {
    using L = TcSmem<D>;
    const int rpad = (int)round_up(q.r, kTcRC);
    __nv_bfloat16* B2h = static_cast<__nv_bfloat16*>(b2ws);
    __nv_bfloat16* B2l = B2h + (size_t)q.BH * L::NE * rpad;
    b2_prep_kernel<D><<<dim3((unsigned)ceil_div(rpad, 128), L::NE, (unsigned)q.BH), 128, 0, st>>>(
        q.V_S, q.w, q.rank, q.r, rpad, B2h, B2l);
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::total);
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc: smem attribute");
    attend_tc_kernel<D><<<dim3((unsigned)ceil_div(q.m, 128), (unsigned)q.BH), kTcThreads, L::total, st>>>(
        static_cast<const __nv_bfloat16*>(q.Q), static_cast<const __nv_bfloat16*>(q.K_S), B2h, B2l, q.m, q.r, rpad,
        q.rank, q.beta, q.vmin, q.vmax, MQ, q.O, g_force_timeout_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc launch");
    return Status::ok();
}

}  // namespace

bool attend_tc_supported(int dtype, int d) { return dtype == 1 && (d == 64 || d == 128); }

size_t attend_tc_scratch_bytes(int64_t BH, int d, int r) {
    const int64_t rpad = round_up(r, kTcRC);
    return 2 * sizeof(__nv_bfloat16) * (size_t)BH * (d + 16) * rpad;
}

Status launch_attend_tc(const AttendRequest& q, const float* MQ, void* b2ws, cudaStream_t st) {
    switch (q.d) {
        case 64: return run_tc<64>(q, MQ, b2ws, st);
        case 128: return run_tc<128>(q, MQ, b2ws, st);
    }
    return Status::fail(2, "attend_tc: unsupported head dim");
}

void set_attend_force_timeout(unsigned long long ns) { g_force_timeout_ns = ns; }

int read_device_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
    }
    return v;
}

}  // namespace wildcat
