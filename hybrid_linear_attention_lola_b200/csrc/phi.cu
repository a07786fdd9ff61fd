// Feature map phi(x) = [softmax(x W), softmax(-x W)] (the low-rank positive
// feature map of LoLA's linear attention, gist.science technical summary,
// "Probleemstelling"; the two-sided softmax form is this engine's fixed choice),
// and state initialisation.
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {

// Blocks with blockIdx.y = w take the rows of kv-head w when every kv-head has its
// own W (gridDim.y = n_kv_heads), all rows otherwise (gridDim.y = 1).
template <typename T>
__global__ void __launch_bounds__(256) phi_kv_kernel(Dims dm, KVSrc<T> src, const float *__restrict__ W,
                                                     int nS, int n, int nvrows,
                                                     T *__restrict__ phi_out)
{
    extern __shared__ float sm[];
    float *Ws = sm;                                   // [d][Dh]
    float *xs = sm + dm.d * dm.Dh + (threadIdx.x >> 5) * dm.d;
    const int hw = blockIdx.y;
    const float *Wh = W + (size_t)hw * dm.d * dm.Dh;
    for (int e = threadIdx.x; e < dm.d * dm.Dh; e += blockDim.x) Ws[e] = Wh[e];
    __syncthreads();
    const int per_stream = nS + dm.R + n;
    const int nsw = gridDim.y > 1 ? dm.B : dm.ns;     // streams this block row covers
    const long long total = (long long)nsw * per_stream;
    const int warps = blockDim.x >> 5;
    for (long long r = (long long)blockIdx.x * warps + (threadIdx.x >> 5); r < total;
         r += (long long)gridDim.x * warps) {
        const int sw = (int)(r / per_stream);
        const int st = gridDim.y > 1 ? sw * dm.Hkv + hw : sw;
        const int i = (int)(r % per_stream);
        const int vrow = i < nS ? i : dm.lam + (i - nS);
        phi_row_warp<T, T>(src.krow(st, vrow), Ws, xs, dm.d, dm.Dh,
                        phi_out + ((size_t)st * nvrows + vrow) * dm.D);
    }
}

// rows: query rows [..][Hq][d]; with gridDim.y = n_kv_heads, blocks of row w take the
// query heads of kv-head w (their own W), else every row (gridDim.y = 1)
template <typename T>
__global__ void __launch_bounds__(256) phi_q_kernel(int d, int Dh, int Hq, int g, const float *__restrict__ W,
                                                    const T *__restrict__ q, long long rows,
                                                    T *__restrict__ phi_out)
{
    extern __shared__ float sm[];
    float *Ws = sm;
    float *xs = sm + d * Dh + (threadIdx.x >> 5) * d;
    const int hw = blockIdx.y;
    const float *Wh = W + (size_t)hw * d * Dh;
    for (int e = threadIdx.x; e < d * Dh; e += blockDim.x) Ws[e] = Wh[e];
    __syncthreads();
    const int warps = blockDim.x >> 5;
    const long long mine = gridDim.y > 1 ? rows / Hq * g : rows;
    for (long long rr = (long long)blockIdx.x * warps + (threadIdx.x >> 5); rr < mine;
         rr += (long long)gridDim.x * warps) {
        const long long r = gridDim.y > 1 ? (rr / g) * Hq + (long long)hw * g + rr % g : rr;
        phi_row_warp<T, T>(q + (size_t)r * d, Ws, xs, d, Dh, phi_out + (size_t)r * 2 * Dh);
    }
}

static int grid_for(long long rows, int warps_per_block)
{
    long long g = (rows + warps_per_block - 1) / warps_per_block;
    if (g > 148 * 16) g = 148 * 16;
    return (int)(g < 1 ? 1 : g);
}

void launch_phi_kv(const Dims &dm, const DevState &S, const void *kin, long long call_start,
                   int n, int nvrows, int /*row_begin_call*/, void *phi_out, int nS,
                   cudaStream_t stream)
{
    const size_t smem = sizeof(float) * ((size_t)dm.d * dm.Dh + 8 * dm.d);
    const long long rows = (long long)dm.ns * (nS + dm.R + n);
    const dim3 grid(grid_for(rows / dm.nW, 8), dm.nW);
    if (dm.dtype == 0) {
        cudaFuncSetAttribute(phi_kv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        KVSrc<float> src{(const float *)S.KS, (const float *)S.VS, (const float *)S.KR,
                         (const float *)S.VR, (const float *)kin, nullptr,
                         dm.lam, dm.R, n, dm.Hkv, dm.d, call_start};
        phi_kv_kernel<float><<<grid, 256, smem, stream>>>(dm, src, S.W, nS, n, nvrows,
                                                          (float *)phi_out);
    } else {
        cudaFuncSetAttribute(phi_kv_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        KVSrc<__nv_bfloat16> src{(const __nv_bfloat16 *)S.KS, (const __nv_bfloat16 *)S.VS,
                                 (const __nv_bfloat16 *)S.KR, (const __nv_bfloat16 *)S.VR,
                                 (const __nv_bfloat16 *)kin, nullptr,
                                 dm.lam, dm.R, n, dm.Hkv, dm.d, call_start};
        phi_kv_kernel<__nv_bfloat16><<<grid, 256, smem, stream>>>(dm, src, S.W, nS, n, nvrows,
                                                                  (__nv_bfloat16 *)phi_out);
    }
}

void launch_phi_q(const Dims &dm, const float *W, const void *q, long long rows, void *phi_out,
                  cudaStream_t stream)
{
    const size_t smem = sizeof(float) * ((size_t)dm.d * dm.Dh + 8 * dm.d);
    const dim3 grid(grid_for(rows / dm.nW, 8), dm.nW);
    if (dm.dtype == 0) {
        cudaFuncSetAttribute(phi_q_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        phi_q_kernel<float><<<grid, 256, smem, stream>>>(dm.d, dm.Dh, dm.Hq, dm.g, W, (const float *)q, rows,
                                                         (float *)phi_out);
    } else {
        cudaFuncSetAttribute(phi_q_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        phi_q_kernel<__nv_bfloat16><<<grid, 256, smem, stream>>>(
            dm.d, dm.Dh, dm.Hq, dm.g, W, (const __nv_bfloat16 *)q, rows, (__nv_bfloat16 *)phi_out);
    }
}

// ---------------------------------------------------------------- init

template <typename T>
__global__ void init_state_kernel(Dims dm, DevState S, const T *__restrict__ W)
{
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long nH = (long long)dm.ns * dm.D * dm.d;
    for (long long e = tid; e < nH; e += stride) S.H[e] = 0.f;
    for (long long e = tid; e < (long long)dm.ns * dm.D; e += stride) S.s[e] = 0.f;
    for (long long e = tid; e < (long long)dm.ns * dm.lam; e += stride) S.idxS[e] = -1;
    for (long long e = tid; e < (long long)dm.ns * dm.Lmax; e += stride) S.pend[e] = 0;
    // cache slots start at zero: tiled loads of aligned 32-slot blocks read the
    // not yet filled slots of a block too (with zero weight)
    const long long nS_ = (long long)dm.ns * dm.lam * dm.d;
    T *KS = (T *)S.KS, *VS = (T *)S.VS;
    for (long long e = tid; e < nS_; e += stride) {
        KS[e] = from_f<T>(0.f);
        VS[e] = from_f<T>(0.f);
    }
    const long long nR = (long long)dm.ns * dm.R * dm.d;
    T *KR = (T *)S.KR, *VR = (T *)S.VR;
    for (long long e = tid; e < nR; e += stride) {
        KR[e] = from_f<T>(0.f);
        VR[e] = from_f<T>(0.f);
    }
    if (W != nullptr) {
        // nW matrices [d][Dh] (one per kv-head, or one shared): fp32 copy and transpose
        T *Wt = (T *)S.Wt;
        const long long per = (long long)dm.d * dm.Dh;
        for (long long e = tid; e < per * dm.nW; e += stride) {
            S.W[e] = to_f<T>(W[e]);
            const long long h = e / per, r = e - h * per;
            const long long a = r / dm.Dh, i = r - a * dm.Dh;
            Wt[h * per + i * dm.d + a] = W[e];
            // the same W^T as a K-major operand image (Dh rows, d columns, 128-byte
            // swizzle): one bulk copy puts it in shared memory ready for the tensor core
            if (S.WtImg != nullptr)
                ((T *)S.WtImg)[h * per + umma::kmajor_offset((int)i, (int)a, dm.Dh) / 2] = W[e];
        }
    }
    if (tid < 4) S.err[tid] = 0;
    for (long long e = tid; e < dm.ns; e += stride) S.dec_cnt[e] = 0;
    // the segment counts only grow (the host keeps the value each wait expects): zeroed
    // when the state is created, never by a reset
    if (W != nullptr && S.seg_done != nullptr)
        for (long long e = tid; e < kMaxSegments; e += stride) S.seg_done[e] = 0;
}

void launch_init_state(const Dims &dm, const DevState &S, const void *W, cudaStream_t stream)
{
    if (dm.dtype == 0)
        init_state_kernel<float><<<148 * 4, 256, 0, stream>>>(dm, S, (const float *)W);
    else
        init_state_kernel<__nv_bfloat16><<<148 * 4, 256, 0, stream>>>(dm, S,
                                                                      (const __nv_bfloat16 *)W);
}

}  // namespace lola
