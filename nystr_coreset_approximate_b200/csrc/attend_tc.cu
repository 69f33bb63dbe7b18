// attend_tc.cu -- weighted-coreset attention on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2 plug-in
// estimator and Alg. 3 WtdAttn, for bfloat16 inputs:
//     P = exp(beta Q K_S^T - beta M_Q),   N = P [V_S | w],   O = clip(N_v / N_w).
//
// One CTA (256 threads; two per query row, splitting its columns) per tile
// of 128 queries of one instance.  Per chunk
// of 64 coreset rows:
//   GEMM1  S = Q K_S^T     tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//                          M = 128, N = 64, K = d
//   exp    the two threads of query row i (TMEM lane i) load their halves
//          of row i of S with tcgen05.ld, form P = exp(beta s - beta M_Q)
//          (one exp2f of an fma; P is rounded to bf16 anyway) and write it as
//          bf16 into shared memory in the UMMA K-major 128-byte-swizzled
//          layout
//   GEMM2  N += P [V_S | w]  with [V_S | w] split as hi + lo bf16 parts (two
//          MMAs), M = 128, N = d + 16, K = 64, accumulated in TMEM across
//          chunks.  The numerator and the denominator use the same rounded P.
// Epilogue: thread i reads its row of N and writes O_i = clip(N_i / N_iw).
//
// Pipeline: the K_S / [V_S|w] chunks go through three shared-memory stages
// (copies two chunks ahead), S has two tensor-memory buffers and P two
// shared-memory buffers, so GEMM1 of chunk c + 1 runs while chunk c is
// exponentiated and the copies of chunk c + 2 land while GEMM2 of chunk c
// runs.  Barrier k of each pair completes once per two chunks; every wait
// names the phase of the chunk it needs, which is always the barrier's most
// recent or next phase.
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
constexpr int kTcThreads = 256;  // two threads per query row: each takes half of the columns
unsigned long long g_force_timeout_ns = 0;  // test hook, 0 = off
constexpr int kTcRC = 64;  // coreset rows per chunk

// NS chunk stages: 3 in general; 2 when the coreset has at most two chunks
// (r <= 128), which the prologue copies at once, so the third stage would
// never be used and its 28-44 KB would keep a second CTA off the SM.
template <int D, int NS = 3>
struct TcSmem {
    static constexpr int NE = D + 16;                           // value columns + w + zero padding
    static constexpr int KB1 = D / 64;                          // 128-byte K blocks of Q / K_S rows
    static constexpr int NSTAGE = NS;                           // K_S / [V_S|w] chunk stages
    static constexpr size_t a1 = 0;                             // Q tile 128 x D
    static constexpr size_t b1_bytes = (size_t)KB1 * kTcRC * 128;  // K_S chunk  RC x D
    static constexpr size_t b2_bytes = (size_t)NE * 128;           // [V_S|w]^T  NE x RC (one 128-byte K block)
    static constexpr size_t stage_bytes = b1_bytes + 2 * b2_bytes;
    static constexpr size_t stages = a1 + (size_t)KB1 * 128 * 128;
    static constexpr size_t a2 = stages + NSTAGE * stage_bytes;   // P, two buffers of 128 x RC
    static constexpr size_t a2_bytes = 128 * 128;
    static constexpr size_t bar = a2 + 2 * a2_bytes;              // 4 mbarriers + TMEM base
    static constexpr size_t total = bar + 64 + 1024;              // + slack for 1024-byte alignment
    static constexpr unsigned tmem_cols = (2 * kTcRC + NE) <= 256 ? 256u : 512u;
};

template <int D, int NS>
__global__ void __launch_bounds__(kTcThreads, 1)
    attend_tc_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K_S,
                     const __nv_bfloat16* __restrict__ B2h, const __nv_bfloat16* __restrict__ B2l, int64_t m, int r,
                     int rpad, const int32_t* __restrict__ rank, float beta, const float* __restrict__ vmin,
                     const float* __restrict__ vmax, const float* __restrict__ MQ, float* __restrict__ O,
                     unsigned long long force_timeout_ns) {
    using L = TcSmem<D, NS>;
    constexpr int NE = L::NE;
    extern __shared__ unsigned char sm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const unsigned sbase = smem_u32(sm);
    const unsigned sA1 = sbase + L::a1;
    uint64_t* mbS = reinterpret_cast<uint64_t*>(sm + L::bar);       // GEMM1 done, per S buffer
    uint64_t* mbG = mbS + 2;                                        // GEMM2 done, per P buffer
    unsigned* tmem_base_slot = reinterpret_cast<unsigned*>(sm + L::bar + 32);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;  // query row (= TMEM lane) and column half
    const int64_t b = blockIdx.y;
    const int64_t i0 = (int64_t)blockIdx.x * 128;
    const int rr = rank[b];
    const int nch = (rr + kTcRC - 1) / kTcRC;
    // P = exp(beta s - beta M_Q) = 2^(s * beta log2 e - beta M_Q log2 e); P is
    // rounded to bf16 (8 significant bits), so exp2f's accuracy is ample
    const float bl2e = beta * 1.4426950408889634f;
    const float sl2e = beta * MQ[b] * 1.4426950408889634f;

    if (tid == 0) {
        for (int k = 0; k < 4; ++k) mbar_init(&mbS[k], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_slot)),
                     "r"(L::tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    auto stage_addr = [&](int st) { return sbase + (unsigned)(L::stages + (size_t)st * L::stage_bytes); };
    // copies of chunk c (rows l0 .. l0 + RC of K_S and of [V_S|w]^T hi / lo) into stage c % 3
    auto load_chunk = [&](int c) {
        const unsigned sb = stage_addr(c % L::NSTAGE);
        const int l0 = c * kTcRC;
        for (int e = tid; e < kTcRC * (D / 8); e += kTcThreads) {
            const int row = e / (D / 8), cc = e % (D / 8);
            const int l = l0 + row;
            const bool ok = l < rr;
            const __nv_bfloat16* src = K_S + ((b * r + (ok ? l : 0)) * (int64_t)D) + cc * 8;
            cp_async16_zfill(sb + (cc >> 3) * (kTcRC * 128) + swz(row, cc & 7), src, ok);
        }
        for (int e = tid; e < NE * (kTcRC / 8); e += kTcThreads) {
            const int row = e / (kTcRC / 8), cc = e % (kTcRC / 8);
            const int64_t off = ((b * NE + row) * (int64_t)rpad) + l0 + cc * 8;
            const unsigned dst = swz(row, cc);
            cp_async16_zfill(sb + L::b1_bytes + dst, B2h + off, true);
            cp_async16_zfill(sb + L::b1_bytes + L::b2_bytes + dst, B2l + off, true);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // Q tile: row `row`, this thread's half of its 16-byte chunks
    {
        const int64_t i = i0 + row;
        const bool ok = i < m;
        const __nv_bfloat16* src = Q + ((b * m + (ok ? i : 0)) * D);
#pragma unroll
        for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c)
            cp_async16_zfill(sA1 + (c >> 3) * (128 * 128) + swz(row, c & 7), src + c * 8, ok);
    }
    if (nch > 0) load_chunk(0);  // committed together with the Q tile
    else asm volatile("cp.async.commit_group;" ::: "memory");
    if (nch > 1) load_chunk(1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tmem = *tmem_base_slot;
    const unsigned tmem_N = tmem + 2 * kTcRC;
    const unsigned lane_off = (unsigned)((warp & 3) * 32) << 16;  // warps w and w + 4 share lanes
    constexpr uint32_t id1 = idesc_bf16(128, kTcRC), id2 = idesc_bf16(128, NE);

    // make the copies of chunk c visible to the tensor cores (all threads)
    auto publish_copies = [&](bool one_more_pending) {
        if (one_more_pending) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };
    auto issue_gemm1 = [&](int c) {
        if (tid == 0) {
            const unsigned sb = stage_addr(c % L::NSTAGE);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const unsigned oa = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                const unsigned ob = (kk >> 2) * (kTcRC * 128) + (kk & 3) * 32;
                mma_bf16(tmem + (c & 1) * kTcRC, umma_desc(sA1 + oa), umma_desc(sb + ob), id1, kk > 0);
            }
            mma_commit(&mbS[c & 1]);
        }
    };

    bool ok = true;
    if (force_timeout_ns) {
        // test hook: wait for a barrier phase that nothing will complete
        const bool w = mbar_wait(&mbG[0], 0, force_timeout_ns);
        if (__syncthreads_or(!w)) ok = false;
    }
    if (ok && nch > 0) {
        publish_copies(nch > 1);
        issue_gemm1(0);
    }
    int c = 0;
    for (; ok && c < nch; ++c) {
        // (1) copies of chunk c + 2 into the stage chunk c - 1 used, once GEMM2(c - 1) has read it
        if (c + 2 < nch) {
            if (c >= 1) {
                const bool w = mbar_wait(&mbG[(c - 1) & 1], ((c - 1) >> 1) & 1);
                if (__syncthreads_or(!w)) { ok = false; break; }
            }
            load_chunk(c + 2);
        }
        // (2) GEMM1 of chunk c + 1 runs on the tensor cores while this chunk is exponentiated
        if (c + 1 < nch) {
            publish_copies(c + 2 < nch);
            issue_gemm1(c + 1);
        }
        // (3) P = exp(beta s - beta M_Q) of chunk c, rounded once to bf16
        const bool w1 = mbar_wait(&mbS[c & 1], (c >> 1) & 1);
        if (__syncthreads_or(!w1)) { ok = false; break; }
        tc_fence_after();
        constexpr int HC = kTcRC / 2;  // columns per thread
        uint32_t pk[HC / 2];
#pragma unroll
        for (int c0 = 0; c0 < HC; c0 += 16) {
            float v[16];
            tmem_ld16(tmem + (c & 1) * kTcRC + lane_off + half * HC + c0, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int l = c * kTcRC + half * HC + c0 + 2 * k;
                const float p0 = l < rr ? exp2f(fmaf(v[2 * k], bl2e, -sl2e)) : 0.f;
                const float p1 = l + 1 < rr ? exp2f(fmaf(v[2 * k + 1], bl2e, -sl2e)) : 0.f;
                const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                pk[c0 / 2 + k] = *reinterpret_cast<const uint32_t*>(&h);
            }
        }
        if (c >= 2) {  // GEMM2(c - 2) has finished reading this P buffer
            const bool w = mbar_wait(&mbG[c & 1], ((c - 2) >> 1) & 1);
            if (__syncthreads_or(!w)) { ok = false; break; }
        }
        unsigned char* pa = sm + L::a2 + (c & 1) * L::a2_bytes;
#pragma unroll
        for (int cc = 0; cc < HC / 8; ++cc)
            *reinterpret_cast<uint4*>(pa + swz(row, half * (HC / 8) + cc)) =
                make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // (4) GEMM2: N += P [V_S|w] (hi and lo parts)
        if (tid == 0) {
            const unsigned sA2 = sbase + (unsigned)(L::a2 + (c & 1) * L::a2_bytes);
            const unsigned sb = stage_addr(c % L::NSTAGE) + (unsigned)L::b1_bytes;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
                for (int kk = 0; kk < kTcRC / 16; ++kk)
                    mma_bf16(tmem_N, umma_desc(sA2 + kk * 32), umma_desc(sb + part * L::b2_bytes + kk * 32), id2,
                             (c > 0 || part > 0 || kk > 0) ? 1 : 0);
            }
            mma_commit(&mbG[c & 1]);
        }
    }
    if (ok && nch > 0) {  // the last GEMM2 before reading N
        const bool w = mbar_wait(&mbG[(nch - 1) & 1], ((nch - 1) >> 1) & 1);
        if (__syncthreads_or(!w)) ok = false;
        tc_fence_after();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // -- epilogue: O = clip(N_v / N_w).  tcgen05.ld is warp-collective, so
    //    every lane loads; only the stores depend on the row being < m. --
    const int64_t i = i0 + row;
    const bool row_ok = i < m;
    if (ok) {
        float* o = O + (b * m + (row_ok ? i : 0)) * D;
        const float* lo = vmin + b * D;
        const float* hi = vmax + b * D;
        if (rr == 0) {
            if (row_ok)
                for (int c2 = half * (D / 2); c2 < (half + 1) * (D / 2); ++c2) o[c2] = lo[c2];  // 0/0 -> v_min
        } else {
            float wv[16];
            tmem_ld16(tmem_N + lane_off + D, wv);
            const float den = wv[0];
#pragma unroll 1
            for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 16) {
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
    } else {
        if (tid == 0) atomicExch(&g_device_status, 5);
        // give issued tensor-core work one more bounded chance to retire
        if (nch > 0 && !force_timeout_ns) {
            mbar_wait(&mbS[0], 0, 100000000ull);
            mbar_wait(&mbG[0], 0, 100000000ull);
        }
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

template <int D, int NS>
cudaError_t launch_tc_kernel(const AttendRequest& q, const float* MQ, const __nv_bfloat16* B2h,
                             const __nv_bfloat16* B2l, int rpad, cudaStream_t st) {
    using L = TcSmem<D, NS>;
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<D, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::total);
    if (e != cudaSuccess) return e;
    attend_tc_kernel<D, NS><<<dim3((unsigned)ceil_div(q.m, 128), (unsigned)q.BH), kTcThreads, L::total, st>>>(
        static_cast<const __nv_bfloat16*>(q.Q), static_cast<const __nv_bfloat16*>(q.K_S), B2h, B2l, q.m, q.r, rpad,
        q.rank, q.beta, q.vmin, q.vmax, MQ, q.O, g_force_timeout_ns);
    return cudaGetLastError();
}

template <int D>
Status run_tc(const AttendRequest& q, const float* MQ, void* b2ws, cudaStream_t st) {
    using L = TcSmem<D>;
    const int rpad = (int)round_up(q.r, kTcRC);
    __nv_bfloat16* B2h = static_cast<__nv_bfloat16*>(b2ws);
    __nv_bfloat16* B2l = B2h + (size_t)q.BH * L::NE * rpad;
    b2_prep_kernel<D><<<dim3((unsigned)ceil_div(rpad, 128), L::NE, (unsigned)q.BH), 128, 0, st>>>(
        q.V_S, q.w, q.rank, q.r, rpad, B2h, B2l);
    // ranks never exceed r, so r <= 2 chunks bounds every instance's chunk count
    cudaError_t e = q.r <= 2 * kTcRC ? launch_tc_kernel<D, 2>(q, MQ, B2h, B2l, rpad, st)
                                     : launch_tc_kernel<D, 3>(q, MQ, B2h, B2l, rpad, st);
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc launch");
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
