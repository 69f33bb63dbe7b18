// Probe of the tensor-core rate per MMA shape (measurement, not a test of
// the method): one thread per SM issues 32 back-to-back GEMMs of 8
// tcgen05.mma kind::f16 instructions (K = 16 each, bf16 operands of zeros,
// fp32 accumulator in tensor memory) and records clock64 after each GEMM's
// issue and after the completion barrier.  Forms: both operands in shared
// memory (SS) or A in tensor memory (TS); N = 64, 128, 256 with M = 128; a
// commit-and-wait after every GEMM; and three other warps reading tensor
// memory meanwhile.  The issuing thread blocks while the tensor pipe is
// full, so cycles per MMA is the pipe's rate for that shape.  Every wait is
// bounded; operands and accumulators stay inside the buffers checked below.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../../nystr_coreset_approximate_b200/csrc/tc_common.cuh"
using namespace wildcat::tc;

constexpr int G = 32;
__device__ long long g_t[148][G + 2];
__device__ int g_ok[148];

__global__ void __launch_bounds__(128, 1) probe(int mode) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ unsigned tbase;
    __shared__ volatile int stop;
    const int tid = threadIdx.x, warp = tid >> 5;
    // operands (A 32 KB, then B up to 64 KB, zeroed) at the first 1024-byte
    // boundary of the 120 KB buffer (so one CTA per SM)
    unsigned char* op = sm + ((1024u - (smem_u32(sm) & 1023u)) & 1023u);
    for (int i = tid; i < 98304 / 16; i += 128) reinterpret_cast<int4*>(op)[i] = make_int4(0, 0, 0, 0);
    if (tid == 0) { mbar_init(&bar, 1); stop = 0; asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tbase)), "r"(512) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tm = tbase;
    const unsigned sbase = smem_u32(op);
    const bool aligned = (sbase & 1023u) == 0;
    if (tid == 0) {
        bool ok = aligned;
        if (ok) {
            const uint64_t da = umma_desc(sbase), db = umma_desc(sbase + 32768);
            const uint32_t hi = (uint32_t)(da >> 32), a_lo = (uint32_t)da, b_lo = (uint32_t)db;
            g_t[blockIdx.x][0] = clock64();
            for (int g = 0; g < G; ++g) {
                const bool ss = mode == 0 || mode == 5 || mode == 7 || ((mode == 2 || mode == 4) && (g & 1) == 0);
                const int N = (mode == 5 || mode == 6) ? 256 : mode == 7 ? 64 : 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t oa = (uint32_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
                    // B: N rows of 128-byte K blocks; two K blocks of N rows each
                    const uint32_t ob = (uint32_t)(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4);
                    if (ss)
                        mma_bf16_w(tm + (N == 256 ? 0 : 256), a_lo + oa, hi, b_lo + ob, hi, idesc_bf16(128, N), kk > 0);
                    else
                        mma_bf16_ts_w(tm, tm + 384 + kk * 8, b_lo + ob, hi, idesc_bf16(128, N), kk > 0);
                }
                if (mode == 3) {  // commit and wait after every GEMM
                    mma_commit(&bar);
                    ok = mbar_wait(&bar, (unsigned)g & 1u, 100000000ull);
                    if (!ok) break;
                }
                g_t[blockIdx.x][1 + g] = clock64();
            }
            if (ok && mode != 3) {
                mma_commit(&bar);
                ok = mbar_wait(&bar, 0, 100000000ull);
            }
            g_t[blockIdx.x][G + 1] = clock64();
        }
        g_ok[blockIdx.x] = ok ? 1 : 0;
        stop = 1;
    } else if (mode == 4 && warp > 0) {
        // other warps keep reading their lane quadrant of columns 128..255 (not touched by the MMAs)
        uint32_t r[32];
        const unsigned ta = tm + ((unsigned)(warp * 32) << 16) + 128;
        float acc = 0.f;
        for (int it = 0; it < 100000 && !stop; ++it) {
            tmem_ld32_nowait(ta + 32 * (it & 3), r);
            tmem_wait_ld();
            acc += __uint_as_float(r[it & 31]);
        }
        if (acc == 12345.f) g_ok[blockIdx.x] = 2;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
    }
}

int main() {
    cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024);
    const char* names[8] = {"SS only", "TS only", "SS/TS alternating", "SS, commit+wait each", "SS/TS + 3 warps tcgen05.ld",
                            "SS N=256", "TS N=256", "SS N=64"};
    for (int mode = 0; mode < 8; ++mode) {
        for (int rep = 0; rep < 2; ++rep) {
            probe<<<148, 128, 120 * 1024>>>(mode);
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
        }
        long long t[148][G + 2]; int ok[148];
        cudaMemcpyFromSymbol(t, g_t, sizeof(t));
        cudaMemcpyFromSymbol(ok, g_ok, sizeof(ok));
        int nok = 0; for (int i = 0; i < 148; ++i) nok += ok[i] == 1;
        long long* a = t[0];
        printf("%-28s ok=%d  issue per GEMM (8 MMAs):", names[mode], nok);
        for (int g = 1; g <= 8; ++g) printf(" %lld", a[g] - a[g - 1]);
        printf(" ... last %lld | all issued %lld | done %lld cycles => %.1f cycles per MMA\n", a[G] - a[G - 1], a[G] - a[0], a[G + 1] - a[0], (double)(a[G + 1] - a[0]) / (G * 8));
    }
    return 0;
}
