// Token-by-token output of a LoLA hybrid-attention layer (gist.science
// technical summary, "Inferentiestrategie": the same combination of linear,
// sparse-cache and sliding-window attention, one query per sequence per call).
//
// The key set of query p inside the open interval [t0, t1):
//   * every cache slot (softmax);
//   * window/ring tokens j in [max(0, t0 - eta), p]:
//       j left the window this interval and was kept   -> already a cache slot, skipped
//       j left the window this interval and was folded -> linear phi(q).phi(k_j) once
//                                                         j <= p - eta, softmax before
//       otherwise                                      -> softmax (inside the window)
//   * the readout phi(q)^T H', phi(q)^T s' of the state.
// The cache and band keys are split over `nsplit` CTAs per stream; each writes
// a partial (m, l, linear den, softmax and linear numerators) and the merge
// kernel combines them with the online-softmax identity and adds the readout.
#include "lola_internal.cuh"

namespace lola {

namespace {

constexpr int KT = 32;
constexpr int DW = 4;  // warps per decode CTA

template <typename T>
__global__ void append_kernel(Dims dm, DevState S, const T *__restrict__ k, const T *__restrict__ v,
                              long long pos)
{
    const int st = blockIdx.x;
    const int slot = (int)(pos & (dm.R - 1));
    T *KR = (T *)S.KR + ((size_t)st * dm.R + slot) * dm.d;
    T *VR = (T *)S.VR + ((size_t)st * dm.R + slot) * dm.d;
    for (int c = threadIdx.x; c < dm.d; c += blockDim.x) {
        KR[c] = k[(size_t)st * dm.d + c];
        VR[c] = v[(size_t)st * dm.d + c];
    }
}

template <typename T>
__global__ void __launch_bounds__(DW * 32)
    decode_attn_kernel(Dims dm, DevState S, DecodeArgs a)
{
    const int split = blockIdx.x, st = blockIdx.y;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const int d = dm.d, D = dm.D, g = dm.g, lam = dm.lam, R = dm.R;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ndu = d >> 5;
    const float scale = rsqrtf((float)d);

    extern __shared__ __align__(16) float sm[];
    float *qs = sm;                  // [g][d]
    float *phq = qs + g * d;         // [g][D]
    float *Ks = phq + g * D;         // [KT][d + 1]
    float *Vs = Ks + KT * (d + 1);   // [KT][d]
    float *phk = Vs + KT * d;        // [KT][D + 1]
    int *ktok = (int *)(phk + KT * (D + 1));
    int *kinfo = ktok + KT;          // 0 soft-if-causal, 1 folded, 2 skip
    int *krow = kinfo + KT;          // row: < lam cache slot, else lam + ring slot

    const T *q = (const T *)a.q;
    for (int e = tid; e < g * d; e += blockDim.x) {
        const int r = e / d, c = e - r * d;
        qs[e] = to_f<T>(q[((size_t)b * dm.Hq + hk * g + r) * d + c]) * scale;
    }
    for (int e = tid; e < g * D; e += blockDim.x) {
        const int r = e / D, i = e - r * D;
        phq[e] = to_f<T>(((const T *)S.phiQd)[((size_t)b * dm.Hq + hk * g + r) * D + i]);
    }

    const long long p = a.pos;
    const long long jlo = a.t0 - dm.eta > 0 ? a.t0 - dm.eta : 0;
    const long long nband = p - jlo + 1;
    const long long nkeys = a.nS + nband;
    const long long ntiles = (nkeys + KT - 1) / KT;
    const long long per = (ntiles + dm.nsplit - 1) / dm.nsplit;
    const long long tb = split * per, te = min(ntiles, tb + per);

    float m[2] = {0.f, 0.f}, l[2] = {0.f, 0.f}, ld[2] = {0.f, 0.f};
    float nsm[2][4] = {}, nln[2][4] = {};
    const T *KS = (const T *)S.KS + (size_t)st * lam * d;
    const T *VS = (const T *)S.VS + (size_t)st * lam * d;
    const T *KR = (const T *)S.KR + (size_t)st * R * d;
    const T *VR = (const T *)S.VR + (size_t)st * R * d;
    const T *phiV = (const T *)S.phiV + (size_t)st * (lam + R) * D;

    for (long long tile = tb; tile < te; ++tile) {
        __syncthreads();
        const long long kb = tile * KT;
        const int nk = (int)min((long long)KT, nkeys - kb);
        if (tid < KT) {
            int tok = -1, info = 2, row = 0;
            if (tid < nk) {
                const long long kk = kb + tid;
                if (kk < a.nS) {
                    row = (int)kk;
                    tok = S.idxS[(size_t)st * lam + kk];
                    info = 0;
                } else {
                    const long long j = jlo + (kk - a.nS);
                    tok = (int)j;
                    row = lam + (int)(j & (R - 1));
                    if (j >= a.L_lo && j < a.L_hi)
                        info = S.pend[(size_t)st * dm.Lmax + (int)(j - a.L_lo)] ? 1 : 2;
                    else
                        info = 0;
                }
            }
            ktok[tid] = tok;
            kinfo[tid] = info;
            krow[tid] = row;
        }
        __syncthreads();
        for (int e = tid; e < nk * d; e += blockDim.x) {
            const int j = e / d, c = e - j * d;
            const int row = krow[j];
            const T *kr = row < lam ? KS + (size_t)row * d : KR + (size_t)(row - lam) * d;
            const T *vr = row < lam ? VS + (size_t)row * d : VR + (size_t)(row - lam) * d;
            Ks[j * (d + 1) + c] = to_f<T>(kr[c]);
            Vs[j * d + c] = to_f<T>(vr[c]);
        }
        for (int e = tid; e < nk * D; e += blockDim.x) {
            const int j = e / D, i = e - j * D;
            if (kinfo[j] == 1) phk[j * (D + 1) + i] = to_f<T>(phiV[(size_t)krow[j] * D + i]);
        }
        __syncthreads();
        const int mytok = lane < nk ? ktok[lane] : -1;
        const int myinfo = lane < nk ? kinfo[lane] : 2;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = warp + DW * rr;
            if (r >= g) continue;
            int cls = 0;  // 0 none, 1 soft, 2 linear
            if (lane < nk && myinfo != 2 && mytok <= p)
                cls = (myinfo == 1 && mytok <= p - dm.eta) ? 2 : 1;
            float sc = -INFINITY;
            if (cls == 1) {
                const float *qr = qs + r * d;
                const float *kr = Ks + lane * (d + 1);
                float dot = 0.f;
                for (int c = 0; c < d; ++c) dot = fmaf(qr[c], kr[c], dot);
                sc = dot;
            }
            const float tmax = warp_max(sc);
            if (tmax > m[rr]) {
                const float f = __expf(m[rr] - tmax);
                l[rr] *= f;
#pragma unroll
                for (int w = 0; w < 4; ++w) nsm[rr][w] *= f;
                m[rr] = tmax;
            }
            const float pw = cls == 1 ? __expf(sc - m[rr]) : 0.f;
            l[rr] += warp_sum(pw);
            float lw = 0.f;
            if (cls == 2) {
                const float *pq = phq + r * D;
                const float *pk = phk + lane * (D + 1);
                float dot = 0.f;
                for (int i = 0; i < D; ++i) dot = fmaf(pq[i], pk[i], dot);
                lw = dot;
            }
            ld[rr] += warp_sum(lw);
            for (int jj = 0; jj < nk; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, pw, jj);
                const float lj = __shfl_sync(0xffffffffu, lw, jj);
                const float *vr = Vs + jj * d;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (w < ndu) {
                        const float vv = vr[lane + 32 * w];
                        nsm[rr][w] = fmaf(pj, vv, nsm[rr][w]);
                        nln[rr][w] = fmaf(lj, vv, nln[rr][w]);
                    }
                }
            }
        }
    }
    // partial record: [m, l, ld, 0, nsm[d], nln[d]]
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int r = warp + DW * rr;
        if (r >= g) continue;
        float *pr = S.part + (((size_t)st * dm.nsplit + split) * g + r) * (2 * d + 4);
        if (lane == 0) {
            pr[0] = m[rr];
            pr[1] = l[rr];
            pr[2] = ld[rr];
            pr[3] = 0.f;
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (w < ndu) {
                pr[4 + lane + 32 * w] = nsm[rr][w];
                pr[4 + d + lane + 32 * w] = nln[rr][w];
            }
        }
    }
}

// One warp per query row: merge the splits, add the state readout, normalise.
template <typename T>
__global__ void decode_merge_kernel(Dims dm, DevState S, void *out_)
{
    const int st = blockIdx.x;
    const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = dm.d, D = dm.D, g = dm.g;
    if (r >= g) return;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const int hq = hk * g + r;
    const int ndu = d >> 5;
    const float *base = S.part + ((size_t)st * dm.nsplit * g + r) * (2 * d + 4);
    const size_t sstride = (size_t)g * (2 * d + 4);
    float M = 0.f;
    for (int sp = 0; sp < dm.nsplit; ++sp) M = fmaxf(M, base[sp * sstride]);
    float L = 0.f, LD = 0.f, nsm[4] = {}, nln[4] = {};
    for (int sp = 0; sp < dm.nsplit; ++sp) {
        const float *pr = base + sp * sstride;
        const float f = __expf(pr[0] - M);
        L = fmaf(f, pr[1], L);
        LD += pr[2];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (w < ndu) {
                nsm[w] = fmaf(f, pr[4 + lane + 32 * w], nsm[w]);
                nln[w] += pr[4 + d + lane + 32 * w];
            }
        }
    }
    // readout phi(q)^T H', phi(q)^T s'
    const T *pq = (const T *)S.phiQd + ((size_t)b * dm.Hq + hq) * D;
    const float *H = S.H + (size_t)st * D * d;
    const float *s = S.s + (size_t)st * D;
    float dd = 0.f;
    for (int i = lane; i < D; i += 32) dd = fmaf(to_f<T>(pq[i]), s[i], dd);
    LD += warp_sum(dd);
    for (int i = 0; i < D; ++i) {
        const float f = to_f<T>(pq[i]);
#pragma unroll
        for (int w = 0; w < 4; ++w)
            if (w < ndu) nln[w] = fmaf(f, H[(size_t)i * d + lane + 32 * w], nln[w]);
    }
    const float em = __expf(-M);
    const float den = L + em * (LD + dm.eps);
    T *out = (T *)out_ + ((size_t)b * dm.Hq + hq) * d;
#pragma unroll
    for (int w = 0; w < 4; ++w)
        if (w < ndu) out[lane + 32 * w] = from_f<T>((nsm[w] + em * nln[w]) / den);
}

__global__ void get_indices_kernel(Dims dm, DevState S, int nS, int32_t *idx, int32_t *cnt)
{
    const long long n = (long long)dm.ns * dm.lam;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x)
        idx[e] = S.idxS[e];
    if (cnt)
        for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < dm.ns;
             e += (long long)gridDim.x * blockDim.x)
            cnt[e] = nS;
}

size_t decode_smem(const Dims &dm)
{
    return sizeof(float) * ((size_t)dm.g * dm.d + (size_t)dm.g * dm.D + KT * (dm.d + 1) +
                            (size_t)KT * dm.d + (size_t)KT * (dm.D + 1)) +
           sizeof(int) * 3 * KT;
}

}  // namespace

void launch_decode_append(const Dims &dm, const DevState &S, const void *k, const void *v,
                          long long pos, cudaStream_t stream)
{
    if (dm.dtype == 0)
        append_kernel<float><<<dm.ns, 128, 0, stream>>>(dm, S, (const float *)k, (const float *)v, pos);
    else
        append_kernel<__nv_bfloat16><<<dm.ns, 128, 0, stream>>>(
            dm, S, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, pos);
}

void launch_decode_attn(const Dims &dm, const DevState &S, const DecodeArgs &a, cudaStream_t stream)
{
    launch_phi_q(dm, S.W, a.q, (long long)dm.B * dm.Hq, S.phiQd, stream);
    const size_t smem = decode_smem(dm);
    dim3 grid(dm.nsplit, dm.ns);
    if (dm.dtype == 0) {
        cudaFuncSetAttribute(decode_attn_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        decode_attn_kernel<float><<<grid, DW * 32, smem, stream>>>(dm, S, a);
        decode_merge_kernel<float><<<dm.ns, 32 * dm.g, 0, stream>>>(dm, S, a.out);
    } else {
        cudaFuncSetAttribute(decode_attn_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        decode_attn_kernel<__nv_bfloat16><<<grid, DW * 32, smem, stream>>>(dm, S, a);
        decode_merge_kernel<__nv_bfloat16><<<dm.ns, 32 * dm.g, 0, stream>>>(dm, S, a.out);
    }
}

void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream)
{
    get_indices_kernel<<<64, 256, 0, stream>>>(dm, S, nS, idx, cnt);
}

}  // namespace lola
