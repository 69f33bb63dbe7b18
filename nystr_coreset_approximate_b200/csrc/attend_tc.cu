// attend_tc.cu -- weighted-coreset attention on the sm_100a tensor cores.
//
// "WildCat: Near-Linear Attention in Theory and Practice", Sec. 2 plug-in
// estimator and Alg. 3 WtdAttn, for bfloat16 inputs:
//     P = exp(beta Q K_S^T - beta M_Q),  N = P V_S,  D = P w,  O = clip(N / D)
// with one shift M_Q per instance (every exponent <= 0; it cancels in N / D).
//
// One CTA owns two tiles of 128 queries of one instance and walks the
// coreset in chunks of 128 rows.  Warp roles (10 warps):
//   warp 0     producer: TMA loads of the two Q tiles (once), of each K_S
//              chunk and of each V_S^T chunk plus its slice of w, into
//              128-byte-swizzled shared memory, ring of NS stages per operand
//   warp 1     tensor cores (one thread issues):
//                GEMM1  S_t = Q_t K_S,c^T   tcgen05.mma kind::f16, M = 128,
//                       N = 128, both operands in shared memory, fp32 in TMEM
//                GEMM2  O_t += P_t V_S,c    A operand P_t read from TMEM
//                       (where the softmax threads left it), N = d
//              in the order G2(c,0) G1(c+1,0) G2(c,1) G1(c+1,1): while one
//              tile's scores are exponentiated the other tile's products run
//   warps 2-5  tile 0, warps 6-9 tile 1: thread i of the group owns query row
//              i (= TMEM lane i).  Per chunk it reads its 128 scores with
//              tcgen05.ld, forms P = 2^(s beta log2e - beta M_Q log2e) on the
//              special-function unit, rounds P once to bf16, writes the
//              packed pairs back over the scores (tcgen05.st) for GEMM2 and
//              accumulates D = sum_l P_l w_l in fp32 from the same rounded P.
//              After the last chunk it reads its row of O from TMEM, forms
//              clip(N / D, v_min, v_max), stages it in the freed Q tile and
//              stores it with TMA.
// Tensor memory (512 columns): O_0, O_1 (d columns each), S_0, S_1 (128 each).
// V_S and w are prepared per call: V_S^T rounded to bf16 (its bf16 rounding
// leaves the plug-in estimator within 6.1e-4 of the value range on every
// workload here, against a bound of 2e-2) and w zero-padded, both zero past
// the instance's rank.  Keys at or past the rank get P = 0.
//
// Every mbarrier wait is bounded (2 s) and gives up when another role has
// given up; an expired wait records WILDCAT_ERR_TIMEOUT in the device status
// word, the CTA drains the copies and tensor-core work it issued (bounded),
// frees its tensor memory and returns.  No load uses cluster multicast.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace wildcat {

__device__ int g_device_status = 0;  // WILDCAT_ERR_TIMEOUT when a bounded wait expired

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        else
            cudaGetLastError();
    });
    if (!encode || (reinterpret_cast<uintptr_t>(base) & 15u) || (s1 & 15u) || (s2 & 15u) ||
        b0 * (uint32_t)elem_bytes != 128u)
        return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return encode(map, type, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using namespace tc;

constexpr int kRows = 128;    // queries per tile = TMEM lanes
constexpr int kChunk = 128;   // coreset rows per chunk = N of GEMM1
constexpr int kWarps = 10;    // producer, tensor cores, two softmax warpgroups
constexpr int kThreads = kWarps * 32;
constexpr unsigned long long kDrainNs = 100000000ull;  // 100 ms for work in flight after an abort
unsigned long long g_force_timeout_ns = 0;             // test hook, 0 = off

template <int NS>
struct Bars {
    uint64_t q_full[2];
    uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
    uint64_t s_full[2], p_full[2], o_full[2];
    uint64_t drain, never;
    unsigned tmem_base;
    int abort;
};

template <int D>
struct Cfg {
    static constexpr int NS = D == 128 ? 2 : 4;          // stages per operand ring
    static constexpr int KB = D / 64;                    // 128-byte blocks per Q / K_S row
    static constexpr uint32_t q_bytes = kRows * D * 2;   // one Q tile; also half of the fp32 O tile
    static constexpr uint32_t k_bytes = kChunk * D * 2;  // one K_S chunk
    static constexpr uint32_t v_bytes = D * kChunk * 2;  // one V_S^T chunk
    static constexpr uint32_t w_bytes = kChunk * 4;      // one chunk of w
    static constexpr uint32_t off_q = 0;
    static constexpr uint32_t off_k = off_q + 2 * q_bytes;
    static constexpr uint32_t off_v = off_k + NS * k_bytes;
    static constexpr uint32_t off_w = off_v + NS * v_bytes;
    static constexpr uint32_t off_bar = off_w + NS * w_bytes;
    static constexpr uint32_t total = off_bar + (uint32_t)sizeof(Bars<NS>) + 1024;  // + 1024-byte alignment slack
    static constexpr unsigned tmem_cols = 512;
    static constexpr unsigned col_O = 0;       // O_t at col_O + t * D
    static constexpr unsigned col_S = 2 * D;   // S_t at col_S + t * kChunk
    static_assert(2 * D + 2 * kChunk <= 512, "tensor memory");
    static_assert(total <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ bool group_all(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const float* __restrict__ wpad, int rpad, int64_t m, const int32_t* __restrict__ rank,
                     float beta, const float* __restrict__ vmin, const float* __restrict__ vmax,
                     const float* __restrict__ MQ, unsigned long long force_timeout_ns) {
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ unsigned char sm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const unsigned sbase = smem_u32(sm);
    Bars<NS>* bars = reinterpret_cast<Bars<NS>*>(sm + C::off_bar);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int64_t i0 = (int64_t)blockIdx.x * (2 * kRows);
    const int ntiles = (m - i0) > kRows ? 2 : 1;
    const int rr = rank[b];
    const int nch = (rr + kChunk - 1) / kChunk;

    if (tid == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->q_full[t], 1);
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 4);  // one arrival per warp of the softmax group
            mbar_init(&bars->o_full[t], 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->never, 1);
        bars->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
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
    if (force_timeout_ns) {
        // test hook: a wait on a barrier phase that nothing completes
        if (tid == 0 && !mbar_wait(&bars->never, 0, force_timeout_ns)) {
            bars->abort = 1;
            atomicExch(&g_device_status, 5);
        }
        __syncthreads();
    }
    const bool go = *abort_flag == 0;
    auto give_up = [&]() {
        *abort_flag = 1;
        atomicExch(&g_device_status, 5);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && go && nch > 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            for (int t = 0; t < ntiles; ++t) {
                mbar_expect_tx(&bars->q_full[t], C::q_bytes);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sbase + C::off_q + t * C::q_bytes + kb * (kRows * 128), &tmQ, kb * 64,
                                (int)(i0 + t * kRows), b, &bars->q_full[t]);
            }
            int issued_k = 0, issued_v = 0;
            bool ok = true;
            for (int c = 0; c < nch; ++c) {
                const int s = c % NS;
                const unsigned ph = (unsigned)(c / NS) & 1u;
                if (c >= NS && !(ok = mbar_wait_or_abort(&bars->k_empty[s], ph ^ 1u, abort_flag))) break;
                mbar_expect_tx(&bars->k_full[s], C::k_bytes);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sbase + C::off_k + s * C::k_bytes + kb * (kChunk * 128), &tmK, kb * 64, c * kChunk, b,
                                &bars->k_full[s]);
                ++issued_k;
                if (c >= NS && !(ok = mbar_wait_or_abort(&bars->v_empty[s], ph ^ 1u, abort_flag))) break;
                mbar_expect_tx(&bars->v_full[s], C::v_bytes + C::w_bytes);
#pragma unroll
                for (int j = 0; j < kChunk / 64; ++j)
                    tma_load_3d(sbase + C::off_v + s * C::v_bytes + j * (D * 128), &tmV, c * kChunk + j * 64, 0, b,
                                &bars->v_full[s]);
                bulk_load(sbase + C::off_w + s * C::w_bytes, wpad + (int64_t)b * rpad + (int64_t)c * kChunk,
                          C::w_bytes, &bars->v_full[s]);
                ++issued_v;
            }
            if (!ok) give_up();
            if (*abort_flag) {
                // copies still in flight must land before the CTA's shared memory is released
                for (int t = 0; t < ntiles; ++t) mbar_wait(&bars->q_full[t], 0, kDrainNs);
                for (int c = std::max(0, issued_k - NS); c < issued_k; ++c)
                    mbar_wait(&bars->k_full[c % NS], (unsigned)(c / NS) & 1u, kDrainNs);
                for (int c = std::max(0, issued_v - NS); c < issued_v; ++c)
                    mbar_wait(&bars->v_full[c % NS], (unsigned)(c / NS) & 1u, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- tensor cores
        if (lane == 0 && go && nch > 0) {
            constexpr uint32_t id1 = idesc_bf16(128, kChunk);
            constexpr uint32_t id2 = idesc_bf16(128, D);
            auto gemm1 = [&](int c, int t) {  // S_t = Q_t K_c^T
                const unsigned qa = sbase + C::off_q + t * C::q_bytes;
                const unsigned kb = sbase + C::off_k + (c % NS) * C::k_bytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(tmem + C::col_S + t * kChunk,
                             umma_desc(qa + (kk >> 2) * (kRows * 128) + (kk & 3) * 32),
                             umma_desc(kb + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32), id1, kk > 0);
            };
            auto gemm2 = [&](int c, int t) {  // O_t += P_t V_c (P_t in tensor memory)
                const unsigned vb = sbase + C::off_v + (c % NS) * C::v_bytes;
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    mma_bf16_ts(tmem + C::col_O + t * D, tmem + C::col_S + t * kChunk + kk * 8,
                                umma_desc(vb + (kk >> 2) * (D * 128) + (kk & 3) * 32), id2, (c > 0 || kk > 0) ? 1 : 0);
            };
            bool ok = mbar_wait_or_abort(&bars->k_full[0], 0, abort_flag);
            for (int t = 0; t < ntiles && ok; ++t) {
                if (!(ok = mbar_wait_or_abort(&bars->q_full[t], 0, abort_flag))) break;
                tc_fence_after();
                gemm1(0, t);
                mma_commit(&bars->s_full[t]);
            }
            if (ok) mma_commit(&bars->k_empty[0]);
            for (int c = 0; c < nch && ok; ++c) {
                const int s = c % NS;
                if (!(ok = mbar_wait_or_abort(&bars->v_full[s], (unsigned)(c / NS) & 1u, abort_flag))) break;
                const bool more = c + 1 < nch;
                const int s1 = (c + 1) % NS;
                for (int t = 0; t < ntiles; ++t) {
                    if (!(ok = mbar_wait_or_abort(&bars->p_full[t], (unsigned)c & 1u, abort_flag))) break;
                    tc_fence_after();
                    gemm2(c, t);
                    if (more) {
                        if (t == 0 &&
                            !(ok = mbar_wait_or_abort(&bars->k_full[s1], (unsigned)((c + 1) / NS) & 1u, abort_flag)))
                            break;
                        tc_fence_after();
                        // issued after GEMM2 of the same tile, which has read P_t out of these
                        // columns by the time this product writes them (tcgen05.mma executes
                        // in issue order)
                        gemm1(c + 1, t);
                        mma_commit(&bars->s_full[t]);
                    } else {
                        mma_commit(&bars->o_full[t]);
                    }
                }
                if (!ok) break;
                mma_commit(&bars->v_empty[s]);
                if (more) mma_commit(&bars->k_empty[s1]);
            }
            if (!ok) give_up();
            // every product issued has finished before tensor memory is released
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, kDrainNs);
        }
    } else {
        // ---------------------------------------------- softmax and epilogue
        const int t = (warp - 2) >> 2;
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;       // query row within the tile = TMEM lane
        const unsigned lane_off = (unsigned)(quad * 32) << 16;
        const unsigned tS = tmem + C::col_S + t * kChunk + lane_off;
        const unsigned tO = tmem + C::col_O + t * D + lane_off;
        const float a = beta * 1.4426950408889634f;
        const float sh = beta * MQ[b] * 1.4426950408889634f;
        float dsum[4] = {0.f, 0.f, 0.f, 0.f};
        if (t < ntiles) {
            bool ok = go;
            for (int c = 0; c < nch && ok; ++c) {
                const int s = c % NS;
                bool w = mbar_wait_or_abort(&bars->s_full[t], (unsigned)c & 1u, abort_flag) &&
                         mbar_wait_or_abort(&bars->v_full[s], (unsigned)(c / NS) & 1u, abort_flag);
                ok = __all_sync(0xffffffffu, w);  // tcgen05.ld / st below are warp-collective
                if (!ok) break;
                tc_fence_after();
                const float4* w4 = reinterpret_cast<const float4*>(sm + C::off_w + s * C::w_bytes);
                const int lim = rr - c * kChunk;  // keys of this chunk below the rank
#pragma unroll
                for (int j = 0; j < kChunk / 32; ++j) {
                    uint32_t v[32];
                    tmem_ld32_nowait(tS + 32 * j, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float p0 = ex2_approx(fmaf(__uint_as_float(v[2 * e]), a, -sh));
                        float p1 = ex2_approx(fmaf(__uint_as_float(v[2 * e + 1]), a, -sh));
                        if (lim < kChunk) {
                            const int k0 = 32 * j + 2 * e;
                            p0 = k0 < lim ? p0 : 0.f;
                            p1 = k0 + 1 < lim ? p1 : 0.f;
                        }
                        pk[e] = pack_bf16x2(p0, p1);
                    }
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 ww = w4[8 * j + e4];
                        const uint32_t x0 = pk[2 * e4], x1 = pk[2 * e4 + 1];
                        dsum[0] = fmaf(__uint_as_float(x0 << 16), ww.x, dsum[0]);
                        dsum[1] = fmaf(__uint_as_float(x0 & 0xffff0000u), ww.y, dsum[1]);
                        dsum[2] = fmaf(__uint_as_float(x1 << 16), ww.z, dsum[2]);
                        dsum[3] = fmaf(__uint_as_float(x1 & 0xffff0000u), ww.w, dsum[3]);
                    }
                    tmem_st16(tS + 16 * j, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[t]);
            }
            if (ok && nch > 0) ok = __all_sync(0xffffffffu, mbar_wait_or_abort(&bars->o_full[t], 0, abort_flag));
            if (!ok && lane == 0) give_up();
            // the whole group agrees before the epilogue's group barriers
            ok = group_all(1 + t, ok);
            if (ok) {
                tc_fence_after();
                const float den = (dsum[0] + dsum[1]) + (dsum[2] + dsum[3]);
                const float rcp = 1.0f / den;  // rank 0: 0 * inf = NaN, which the clip turns into v_min
                const float* lo = vmin + (int64_t)b * D;
                const float* hi = vmax + (int64_t)b * D;
                unsigned char* stage = sm + C::off_q + t * C::q_bytes;  // this tile's Q is no longer read
                const unsigned stage_s = sbase + C::off_q + t * C::q_bytes;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
#pragma unroll 1
                    for (int g = 0; g < D / 64; ++g) {
                        const int col0 = h * (D / 2) + g * 32;
                        uint32_t v[32];
                        if (nch > 0) {
                            tmem_ld32_nowait(tO + col0, v);
                            tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k) v[k] = 0u;
                        }
                        unsigned char* box = stage + g * (kRows * 128) + row * 128;
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) {
                            const float4 l4 = __ldg(reinterpret_cast<const float4*>(lo + col0) + cc);
                            const float4 h4 = __ldg(reinterpret_cast<const float4*>(hi + col0) + cc);
                            float4 o;
                            o.x = fminf(fmaxf(__uint_as_float(v[4 * cc + 0]) * rcp, l4.x), h4.x);
                            o.y = fminf(fmaxf(__uint_as_float(v[4 * cc + 1]) * rcp, l4.y), h4.y);
                            o.z = fminf(fmaxf(__uint_as_float(v[4 * cc + 2]) * rcp, l4.z), h4.z);
                            o.w = fminf(fmaxf(__uint_as_float(v[4 * cc + 3]) * rcp, l4.w), h4.w);
                            *reinterpret_cast<float4*>(box + ((cc ^ (row & 7)) << 4)) = o;
                        }
                    }
                    fence_async_smem();
                    named_barrier_sync(1 + t, 128);
                    if (row == 0) {
#pragma unroll
                        for (int g = 0; g < D / 64; ++g)
                            tma_store_3d(&tmO, h * (D / 2) + g * 32, (int)(i0 + t * kRows), b,
                                         stage_s + g * (kRows * 128));
                        bulk_commit();
                        bulk_wait_read_all();
                    }
                    named_barrier_sync(1 + t, 128);
                }
                if (row == 0) bulk_wait_all();
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

// V_S^T rounded to bf16 and w zero-padded to rpad rows, both zero at and past
// the rank: VT[b, c, l] for c < D, l < rpad; wpad[b, l].
template <int D>
__global__ void vt_prep_kernel(const float* __restrict__ V_S, const float* __restrict__ w,
                               const int32_t* __restrict__ rank, int r, int rpad, __nv_bfloat16* __restrict__ VT,
                               float* __restrict__ wpad) {
    __shared__ float tile[32][33];
    const int64_t b = blockIdx.z;
    const int l0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    const int rr = rank[b];
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int l = l0 + k;
        tile[k][threadIdx.x] = l < rr ? V_S[(b * r + l) * (int64_t)D + c0 + threadIdx.x] : 0.f;
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += blockDim.y)
        VT[(b * D + c0 + k) * (int64_t)rpad + l0 + threadIdx.x] = __float2bfloat16_rn(tile[threadIdx.x][k]);
    if (blockIdx.y == 0 && threadIdx.y == 0) {
        const int l = l0 + threadIdx.x;
        wpad[b * rpad + l] = l < rr ? w[b * r + l] : 0.f;
    }
}

template <int D>
Status run_tc(const AttendRequest& q, const float* MQ, void* scratch, cudaStream_t st) {
    using C = Cfg<D>;
    const int rpad = (int)round_up(q.r, kChunk);
    __nv_bfloat16* VT = static_cast<__nv_bfloat16*>(scratch);
    float* wpad = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                           round_up((int64_t)sizeof(__nv_bfloat16) * q.BH * D * rpad, 256));
    vt_prep_kernel<D><<<dim3((unsigned)(rpad / 32), D / 32, (unsigned)q.BH), dim3(32, 8), 0, st>>>(
        q.V_S, q.w, q.rank, q.r, rpad, VT, wpad);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc: prep launch");
    if (q.m == 0) return Status::ok();
    CUtensorMap tmQ, tmK, tmV, tmO;
    const uint64_t BH = (uint64_t)q.BH, m = (uint64_t)q.m, r = (uint64_t)q.r;
    bool ok = make_tmap_3d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.Q, D, m, BH, D * 2ull, m * D * 2ull, 64, kRows) &&
              make_tmap_3d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.K_S, D, r, BH, D * 2ull, r * D * 2ull, 64,
                           kChunk) &&
              make_tmap_3d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, VT, (uint64_t)rpad, D, BH, rpad * 2ull,
                           (uint64_t)D * rpad * 2ull, 64, D) &&
              make_tmap_3d(&tmO, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, q.O, D, m, BH, D * 4ull, m * D * 4ull, 32, kRows);
    if (!ok) return Status::fail(3, "attend_tc: tensor map encoding failed");
    e = cudaFuncSetAttribute(attend_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::total);
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc: shared memory attribute");
    attend_tc_kernel<D><<<dim3((unsigned)ceil_div(q.m, 2 * kRows), (unsigned)q.BH), kThreads, C::total, st>>>(
        tmQ, tmK, tmV, tmO, wpad, rpad, q.m, q.rank, q.beta, q.vmin, q.vmax, MQ, g_force_timeout_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return Status::cuda(e, "attend_tc launch");
    return Status::ok();
}

}  // namespace

bool attend_tc_supported(int dtype, int d) { return dtype == 1 && (d == 64 || d == 128); }

size_t attend_tc_scratch_bytes(int64_t BH, int d, int r) {
    const int64_t rpad = round_up(r, kChunk);
    return (size_t)round_up((int64_t)sizeof(__nv_bfloat16) * BH * d * rpad, 256) + sizeof(float) * (size_t)BH * rpad;
}

Status launch_attend_tc(const AttendRequest& q, const float* MQ, void* scratch, cudaStream_t st) {
    if ((reinterpret_cast<uintptr_t>(q.O) & 15u) || (reinterpret_cast<uintptr_t>(q.Q) & 15u) ||
        (reinterpret_cast<uintptr_t>(q.K_S) & 15u) || (reinterpret_cast<uintptr_t>(q.vmin) & 15u) ||
        (reinterpret_cast<uintptr_t>(q.vmax) & 15u))
        return Status::fail(1, "attend_tc: Q, K_S, O, vmin and vmax must be 16-byte aligned");
    switch (q.d) {
        case 64: return run_tc<64>(q, MQ, scratch, st);
        case 128: return run_tc<128>(q, MQ, scratch, st);
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
