// Test hook for the tensor-core layer: one CTA computes C = A * op(B) with
// tcgen05.mma from operands staged in the same 128-byte-swizzled shared-memory
// layouts the inference kernels use (see umma.cuh), so the descriptor and
// layout conventions are checked against a plain matmul on the device.
#include "../../include/lola.h"
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {
namespace {

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per tensor-core completion wait

__global__ void __launch_bounds__(128)
    umma_selftest_kernel(int layout, const __nv_bfloat16 *__restrict__ A,
                         const __nv_bfloat16 *__restrict__ B, float *__restrict__ C, int N, int K,
                         int *err)
{
    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    const int Kp = (K + 63) / 64 * 64;         // K-major rows span whole 128-byte atoms
    uint8_t *sA = base;                        // [128 x Kp] K-major
    uint8_t *sB = base + 128 * Kp * 2;         // K-major [N x Kp] or MN-major [K x N]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const bool a_mn = layout >= 2;            // layouts 2, 3: A given as [K][128], M contiguous
    if (!a_mn) {
        for (int e = tid; e < 128 * K; e += blockDim.x) {
            const int r = e / K, k = e - r * K;
            *(__nv_bfloat16 *)(sA + umma::kmajor_offset(r, k, 128)) = A[e];
        }
    } else {
        for (int e = tid; e < 128 * K; e += blockDim.x) {
            const int k = e / 128, m = e - k * 128;
            *(__nv_bfloat16 *)(sA + umma::mnmajor_offset(k, m, 128)) = A[e];
        }
    }
    if (layout == 0 || layout == 3) {
        for (int e = tid; e < N * K; e += blockDim.x) {
            const int n = e / K, k = e - n * K;
            *(__nv_bfloat16 *)(sB + umma::kmajor_offset(n, k, N)) = B[e];
        }
    } else {
        for (int e = tid; e < K * N; e += blockDim.x) {
            const int k = e / N, n = e - k * N;
            *(__nv_bfloat16 *)(sB + umma::mnmajor_offset(k, n, N)) = B[e];
        }
    }
    if (tid == 0) umma::mbar_init(&mbar, 1);
    umma::fence_async_smem();
    __syncthreads();
    if (warp == 0) umma::tmem_alloc(&tslot, 256);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t taddr = tslot;
    if (tid == 0) {
        const bool b_mn = layout == 1 || layout == 2;
        const uint32_t id = umma::idesc_bf16(128, N, a_mn, b_mn);
        const uint32_t a0 = umma::smem_u32(sA), b0 = umma::smem_u32(sB);
        for (int ks = 0; ks < K / 16; ++ks) {
            const uint64_t ad = a_mn ? umma::mnmajor_desc(a0, ks, 128) : umma::kmajor_desc(a0, ks, 128);
            const uint64_t bd = b_mn ? umma::mnmajor_desc(b0, ks, N) : umma::kmajor_desc(b0, ks, N);
            umma::mma_ss(taddr, ad, bd, id, ks > 0 ? 1u : 0u);
        }
        umma::mma_commit(&mbar);
    }
    const bool ok = umma::mbar_wait(&mbar, 0, kWaitNs);
    if (!ok && lane == 0) atomicOr(err, ERR_TIMEOUT);
    umma::fence_after_sync();
    if (ok) {
        const int row = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            umma::tmem_ld16(taddr + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) C[(size_t)row * N + c0 + i] = v[i];
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(taddr, 256);
}

}  // namespace
}  // namespace lola

extern "C" lola_status lola_selftest_umma(int layout, const void *A, const void *B, float *C, int N,
                                          int K, int *dev_err, void *cuda_stream)
{
    if (!A || !B || !C || !dev_err || layout < 0 || layout > 3) return LOLA_ERR_INVALID_ARG;
    if (N < 16 || N > 256 || N % 16 || K < 16 || K > 256 || K % 16) return LOLA_ERR_INVALID_ARG;
    if ((layout == 1 || layout == 2) && N % 64) return LOLA_ERR_INVALID_ARG;
    if (layout >= 2 && K % 8) return LOLA_ERR_INVALID_ARG;
    const size_t Kp = (size_t)(K + 63) / 64 * 64;
    const size_t smem = 128 * Kp * 2 + ((layout == 0 || layout == 3) ? (size_t)N * Kp * 2 : (size_t)N * K * 2) + 1024;
    cudaFuncSetAttribute(lola::umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    lola::umma_selftest_kernel<<<1, 128, smem, (cudaStream_t)cuda_stream>>>(
        layout, (const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, C, N, K, dev_err);
    return cudaGetLastError() == cudaSuccess ? LOLA_OK : LOLA_ERR_CUDA;
}
