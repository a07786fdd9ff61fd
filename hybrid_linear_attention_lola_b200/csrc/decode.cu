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
#include "lola_internal.cuh"

namespace lola {

namespace {

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

// ---------------------------------------------------------------- bandwidth-oriented decode
//
// One CTA = 128 keys of one stream (4 warps x 32 keys) plus a slice of the
// state readout; all g query heads of the stream are handled together so each
// key/value row is read once. Scores: one lane per key against the queries in
// shared memory. P V: one lane per value dimension, the key's weight broadcast
// by shuffle, value rows read coalesced. Each CTA writes a partial
// [m, l, linear den, 0, softmax num[d], linear num[d]] per head; the merge
// combines the splits with the online-softmax identity.
constexpr int DT = 128;
constexpr int KPC = 128;

template <typename T, int DPL>
__device__ __forceinline__ void load_row(const T *row, int lane, float (&v)[DPL])
{
#pragma unroll
    for (int u = 0; u < DPL; ++u) v[u] = to_f<T>(row[lane * DPL + u]);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(DT) decode2_kernel(Dims dm, DevState S, DecodeArgs a, int hpc)
{
    constexpr int d = 32 * DPL;
    const int split = blockIdx.x, st = blockIdx.y;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const int D = dm.D, g = dm.g, lam = dm.lam, R = dm.R;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ float qs[8 * d];                  // queries of the group, scaled by 1/sqrt(d)
    __shared__ float phq[8 * 256];               // their features
    __shared__ float red[4][8][3 + 2 * d];       // per-warp partials
    const float scale = rsqrtf((float)d);
    const T *q = (const T *)a.q + ((size_t)b * dm.Hq + (size_t)hk * g) * d;
    const T *pq = (const T *)S.phiQd + ((size_t)b * dm.Hq + (size_t)hk * g) * D;
    for (int e = tid; e < g * d; e += DT) qs[e] = to_f<T>(q[e]) * scale;
    for (int e = tid; e < g * D; e += DT) phq[e] = to_f<T>(pq[e]);
    __syncthreads();

    const long long p = a.pos;
    const long long jlo = a.t0 - dm.eta > 0 ? a.t0 - dm.eta : 0;
    const int nband = (int)(p - jlo + 1);
    const int nkeys = a.nS + nband;
    const int k0 = split * KPC, k1 = min(nkeys, k0 + KPC);
    const T *KS = (const T *)S.KS + (size_t)st * lam * d;
    const T *VS = (const T *)S.VS + (size_t)st * lam * d;
    const T *KR = (const T *)S.KR + (size_t)st * R * d;
    const T *VR = (const T *)S.VR + (size_t)st * R * d;
    const T *phiV = (const T *)S.phiV + (size_t)st * (lam + R) * D;

    float m[8], l[8], ld[8], o[8][DPL], lo[8][DPL];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        m[h] = 0.f;          // the shift never goes below 0
        l[h] = 0.f;
        ld[h] = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) o[h][u] = lo[h][u] = 0.f;
    }

    const int kk0 = k0 + warp * 32;
    if (kk0 < k1) {
        const int key = kk0 + lane;
        const bool valid = key < k1;
        int cls = 0;                    // 0 skip, 1 softmax, 2 linear
        int row = 0;                    // < lam: cache slot; else lam + ring slot
        if (valid) {
            if (key < a.nS) {
                row = key;
                cls = 1;
            } else {
                const long long j = jlo + (key - a.nS);
                row = lam + (int)(j & (R - 1));
                if (j >= a.L_lo && j < a.L_hi)
                    cls = S.pend[(size_t)st * dm.Lmax + (int)(j - a.L_lo)] ? (j <= p - dm.eta ? 2 : 1) : 0;
                else
                    cls = 1;
            }
        }
        const T *krow = row < lam ? KS + (size_t)row * d : KR + (size_t)(row - lam) * d;
        const T *vrow = row < lam ? VS + (size_t)row * d : VR + (size_t)(row - lam) * d;
        // scores of this lane's key for every head
        float sc[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) sc[h] = 0.f;
        if (cls == 1) {
            for (int c0 = 0; c0 < d; c0 += 8) {
                float kf[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) kf[u] = to_f<T>(krow[c0 + u]);
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    if (h < g) {
                        const float *qh = qs + h * d + c0;
#pragma unroll
                        for (int u = 0; u < 8; ++u) sc[h] = fmaf(qh[u], kf[u], sc[h]);
                    }
                }
            }
        }
        float pw[8], wl[8];
        const bool anylin = __any_sync(0xffffffffu, cls == 2);
#pragma unroll
        for (int h = 0; h < 8; ++h) wl[h] = 0.f;
        if (anylin && cls == 2) {
            const T *pk = phiV + (size_t)row * D;
            for (int i = 0; i < D; ++i) {
                const float f = to_f<T>(pk[i]);
#pragma unroll
                for (int h = 0; h < 8; ++h)
                    if (h < g) wl[h] = fmaf(phq[h * D + i], f, wl[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            if (h < g) {
                const float s_ = cls == 1 ? sc[h] : -INFINITY;
                const float mn = fmaxf(m[h], warp_max(s_));
                const float f = __expf(m[h] - mn);
                pw[h] = cls == 1 ? __expf(s_ - mn) : 0.f;
                l[h] = l[h] * f + warp_sum(pw[h]);
#pragma unroll
                for (int u = 0; u < DPL; ++u) o[h][u] *= f;
                m[h] = mn;
                if (anylin) ld[h] += warp_sum(wl[h]);
            } else {
                pw[h] = 0.f;
            }
        }
        // P V over the warp's keys: lane owns value dims [lane*DPL, lane*DPL + DPL)
        const int nvalid = min(32, k1 - kk0);
        const unsigned long long vaddr = (unsigned long long)vrow;
        for (int jj = 0; jj < nvalid; ++jj) {
            const T *vr = (const T *)__shfl_sync(0xffffffffu, vaddr, jj);
            float vf[DPL];
            load_row<T, DPL>(vr, lane, vf);
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (h < g) {
                    const float pj = __shfl_sync(0xffffffffu, pw[h], jj);
#pragma unroll
                    for (int u = 0; u < DPL; ++u) o[h][u] = fmaf(pj, vf[u], o[h][u]);
                    if (anylin) {
                        const float wj = __shfl_sync(0xffffffffu, wl[h], jj);
#pragma unroll
                        for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(wj, vf[u], lo[h][u]);
                    }
                }
            }
        }
    }
    // slice of the readout phi(q)^T H', phi(q)^T s' (unscaled linear sums)
    {
        const float *Hs = S.H + (size_t)st * D * d;
        const float *ss = S.s + (size_t)st * D;
        const int h0 = split * hpc, h1 = min(D, h0 + hpc);
        for (int i = h0 + warp; i < h1; i += 4) {
            float hv[DPL];
            load_row<float, DPL>(Hs + (size_t)i * d, lane, hv);
            const float si = ss[i];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (h < g) {
                    const float f = phq[h * D + i];
#pragma unroll
                    for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(f, hv[u], lo[h][u]);
                    ld[h] = fmaf(f, si, ld[h]);
                }
            }
        }
    }
    // combine the 4 warps, then write this CTA's partial per head
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        if (h < g) {
            if (lane == 0) {
                red[warp][h][0] = m[h];
                red[warp][h][1] = l[h];
                red[warp][h][2] = ld[h];
            }
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                red[warp][h][3 + lane * DPL + u] = o[h][u];
                red[warp][h][3 + d + lane * DPL + u] = lo[h][u];
            }
        }
    }
    __syncthreads();
    for (int h = warp; h < g; h += 4) {
        float M = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, red[w][h][0]);
        float L = 0.f, LD = 0.f, O[DPL], LO[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) O[u] = LO[u] = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float f = __expf(red[w][h][0] - M);
            L = fmaf(f, red[w][h][1], L);
            LD += red[w][h][2];
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                O[u] = fmaf(f, red[w][h][3 + lane * DPL + u], O[u]);
                LO[u] += red[w][h][3 + d + lane * DPL + u];
            }
        }
        float *pr = S.part + (((size_t)st * dm.nsplit + split) * g + h) * (2 * d + 4);
        if (lane == 0) {
            pr[0] = M;
            pr[1] = L;
            pr[2] = LD;
            pr[3] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            pr[4 + lane * DPL + u] = O[u];
            pr[4 + d + lane * DPL + u] = LO[u];
        }
    }
}

// One warp per query head: merge the splits (readout included in the partials).
template <typename T>
__global__ void decode2_merge_kernel(Dims dm, DevState S, void *out_)
{
    const int st = blockIdx.x;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = dm.d, g = dm.g;
    if (h >= g) return;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const float *base = S.part + ((size_t)st * dm.nsplit * g + h) * (2 * d + 4);
    const size_t sstride = (size_t)g * (2 * d + 4);
    float M = 0.f;
    for (int sp = 0; sp < dm.nsplit; ++sp) M = fmaxf(M, base[sp * sstride]);
    float L = 0.f, LD = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f}, LO[4] = {0.f, 0.f, 0.f, 0.f};
    const int dpl = d >> 5;
    for (int sp = 0; sp < dm.nsplit; ++sp) {
        const float *pr = base + sp * sstride;
        const float f = __expf(pr[0] - M);
        L = fmaf(f, pr[1], L);
        LD += pr[2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u < dpl) {
                O[u] = fmaf(f, pr[4 + lane * dpl + u], O[u]);
                LO[u] += pr[4 + d + lane * dpl + u];
            }
        }
    }
    const float em = __expf(-M);
    const float rden = 1.f / (L + em * (LD + dm.eps));
    T *out = (T *)out_ + ((size_t)b * dm.Hq + (size_t)hk * g + h) * d;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (u < dpl) out[lane * dpl + u] = from_f<T>((O[u] + em * LO[u]) * rden);
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
    dim3 grid(dm.nsplit, dm.ns);
    const int hpc = (dm.D + dm.nsplit - 1) / dm.nsplit;
#define LOLA_DECODE2(T, DPL) decode2_kernel<T, DPL><<<grid, DT, 0, stream>>>(dm, S, a, hpc)
    if (dm.dtype == 0) {
        if (dm.d == 32) LOLA_DECODE2(float, 1);
        else if (dm.d == 64) LOLA_DECODE2(float, 2);
        else LOLA_DECODE2(float, 4);
        decode2_merge_kernel<float><<<dm.ns, 32 * dm.g, 0, stream>>>(dm, S, a.out);
    } else {
        if (dm.d == 32) LOLA_DECODE2(__nv_bfloat16, 1);
        else if (dm.d == 64) LOLA_DECODE2(__nv_bfloat16, 2);
        else LOLA_DECODE2(__nv_bfloat16, 4);
        decode2_merge_kernel<__nv_bfloat16><<<dm.ns, 32 * dm.g, 0, stream>>>(dm, S, a.out);
    }
#undef LOLA_DECODE2
}

void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream)
{
    get_indices_kernel<<<64, 256, 0, stream>>>(dm, S, nS, idx, cnt);
}

}  // namespace lola
