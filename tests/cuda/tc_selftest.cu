// GPU self-test of the tcgen05 building blocks in tc_ptx.cuh: one CTA runs a
// single bf16 GEMM D = A * B^T (A: M x K, B: N x K given row-major in global
// memory) through shared-memory descriptors in K-major or MN-major SW128
// tiles, then dumps all 128 TMEM lanes x N columns.  Test infrastructure only.
#include <cstdint>
#include <cuda_runtime.h>

#include "tc_ptx.cuh"

using namespace gdn::ptx;

struct Args {
    const __nv_bfloat16 *A, *B;
    float *D;
    int M, N, Kd, a_mn, b_mn, swap;
    int *err;
    int a_tmem;  // A from TMEM (K-major, packed bf16 pairs) instead of shared memory
};

__device__ __forceinline__ uint64_t desc_mn_variant(uint32_t base, int R, int s, int swap) {
    return swap ? sdesc(base + (uint32_t)(s * 2048), 1024, (uint32_t)(R * 128))
                : desc_mnmajor(base, R, s);
}

__global__ void __launch_bounds__(128, 1) mma_selftest(Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *As = base, *Bs = base + 65536;
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x;
    const int RA = a.a_mn ? a.Kd : a.M;
    for (int e = tid; e < a.M * a.Kd; e += 128) {
        const int m = e / a.Kd, k = e % a.Kd;
        const uint32_t off = a.a_mn ? sw128_off(a.Kd, k, m) : sw128_off(a.M, m, k);
        *(__nv_bfloat16 *)(As + off) = a.A[e];
    }
    for (int e = tid; e < a.N * a.Kd; e += 128) {
        const int n = e / a.Kd, k = e % a.Kd;
        const uint32_t off = a.b_mn ? sw128_off(a.Kd, k, n) : sw128_off(a.N, n, k);
        *(__nv_bfloat16 *)(Bs + off) = a.B[e];
    }
    fence_async_smem();
    if (tid == 0) {
        mbar_init(&mbar, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    constexpr uint32_t kAcol = 256;  // A's columns when it is taken from TMEM
    if (a.a_tmem) {  // thread tid writes row m = tid of A into its lane, bf16 pairs
        const int w = tid / 32;
        for (int c = 0; c < a.Kd / 2; c += 16) {
            uint32_t r[16];
            for (int i = 0; i < 16; ++i) {
                const int k = 2 * (c + i);
                const __nv_bfloat16 lo = tid < a.M ? a.A[(size_t)tid * a.Kd + k] : __float2bfloat16(0.f);
                const __nv_bfloat16 hi = tid < a.M ? a.A[(size_t)tid * a.Kd + k + 1] : __float2bfloat16(0.f);
                r[i] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            }
            tmem_st16(tmem + ((uint32_t)(w * 32) << 16) + kAcol + (uint32_t)c, r);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(a.M, a.N, a.a_mn, a.b_mn);
        const uint32_t sa = smem_u32(As), sb = smem_u32(Bs);
        for (int s = 0; s < a.Kd / 16; ++s) {
            const uint64_t db =
                a.b_mn ? desc_mn_variant(sb, a.Kd, s, a.swap) : desc_kmajor(sb, a.N, s);
            if (a.a_tmem) {
                mma_bf16_ta(tmem, tmem + kAcol + 8u * s, db, idesc, s > 0 ? 1u : 0u);
            } else {
                const uint64_t da =
                    a.a_mn ? desc_mn_variant(sa, RA, s, a.swap) : desc_kmajor(sa, RA, s);
                mma_bf16(tmem, da, db, idesc, s > 0 ? 1u : 0u);
            }
        }
        mma_commit(&mbar);
    }
    const bool ok = mbar_wait(&mbar, 0, 1u << 22);
    if (!ok && (tid & 31) == 0) atomicExch(a.err, 1);
    tc_fence_after();
    const int w = tid / 32;
    for (int c = 0; c < a.N; c += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(w * 32) << 16) + (uint32_t)c, v);
        tmem_ld_wait();
        for (int i = 0; i < 16; ++i) a.D[(size_t)tid * a.N + c + i] = v[i];
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 512);
}

extern "C" int tc_selftest_run(const void *A, const void *B, float *D, int M, int N, int Kd,
                               int a_mn, int b_mn, int swap, int *err_dev, int a_tmem) {
    if (M != 64 && M != 128) return -1;
    if (N < 16 || N > 256 || N % 16 || Kd < 16 || Kd > 128 || Kd % 16) return -1;
    if (a_tmem && (M != 128 || a_mn || Kd % 32)) return -1;
    Args a{(const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, D, M, N, Kd, a_mn, b_mn, swap,
           err_dev, a_tmem};
    const int smem = 65536 * 2 + 1024;
    cudaFuncSetAttribute(mma_selftest, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    mma_selftest<<<1, 128, smem>>>(a);
    cudaError_t e = cudaDeviceSynchronize();
    return (int)e;
}
