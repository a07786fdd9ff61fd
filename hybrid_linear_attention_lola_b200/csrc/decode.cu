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
// One CTA = a range of 32-key chunks of one stream (4 warps, each walking its
// chunks with the next chunk's key/value rows copied into shared memory while
// the current one is processed) plus a slice of the state readout; all g query
// heads of the stream are handled together so each row is read once. Scores:
// one lane per key against the queries in shared memory. P V: one lane per value
// dimension, the key's weight broadcast by shuffle. Each CTA writes a partial
// [m, l, linear den, 0, softmax num[d], linear num[d]] per head; the last CTA of
// the stream (a per-stream counter) merges them with the online-softmax identity.
constexpr int DT = 128;

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))), "l"(gmem)
                 : "memory");
}

template <typename T, int DPL>
__device__ __forceinline__ void load_row(const T *row, int lane, float (&v)[DPL])
{
#pragma unroll
    for (int u = 0; u < DPL; ++u) v[u] = to_f<T>(row[lane * DPL + u]);
}

template <typename T> struct Vec8;   // 16 bytes of T -> 8 (bf16) or 4 (fp32) floats
template <> struct Vec8<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const void *p, float *f)
    {
        const uint4 r = *(const uint4 *)p;
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <> struct Vec8<float> {
    static constexpr int N = 4;
    __device__ static void load(const void *p, float *f)
    {
        const float4 r = *(const float4 *)p;
        f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
    }
};

struct DecodeSmem {
    size_t off_phq, off_rows, off_kv, kstride, vstride, buf_bytes, warp_bytes, total;
};

// [queries fp32 8 x d][features fp32 8 x D][per warp x 2 buffers: row and class of each key]
// [per warp x 2 buffers: 32 padded key rows + 32 value rows]; the per-warp partials of the
// final combine reuse the row buffers.
template <typename T, int DPL>
__host__ __device__ inline DecodeSmem decode_smem_layout(int D)
{
    constexpr int d = 32 * DPL;
    DecodeSmem L{};
    L.off_phq = (size_t)8 * d * 4;
    L.off_rows = L.off_phq + (size_t)8 * D * 4;
    L.off_kv = (L.off_rows + (size_t)4 * 2 * 2 * 32 * 4 + 15) / 16 * 16;
    L.kstride = (size_t)d * sizeof(T) + 16;                // padded against bank conflicts
    L.vstride = (size_t)d * sizeof(T);
    L.buf_bytes = 32 * (L.kstride + L.vstride);
    L.warp_bytes = 2 * L.buf_bytes;
    const size_t kv = 4 * L.warp_bytes;
    const size_t red = (size_t)4 * 8 * (3 + 2 * d) * 4;
    L.total = L.off_kv + (kv > red ? kv : red);
    return L;
}

// Where a key of the decode key list lives and how it is attended.
struct KeyRef {
    int row;   // < lam: cache slot; else lam + ring slot
    int cls;   // 0 skip, 1 softmax, 2 linear
};

__device__ __forceinline__ KeyRef decode_key(const Dims &dm, const DevState &S, const DecodeArgs &a,
                                             int st, int key, int nkeys, long long jlo)
{
    KeyRef k{0, 0};
    if (key >= nkeys) return k;
    if (key < a.nS) {
        k.row = key;
        k.cls = 1;
        return k;
    }
    const long long j = jlo + (key - a.nS);
    k.row = dm.lam + (int)(j & (dm.R - 1));
    if (j >= a.L_lo && j < a.L_hi)
        k.cls = S.pend[(size_t)st * dm.Lmax + (int)(j - a.L_lo)] ? (j <= a.pos - dm.eta ? 2 : 1) : 0;
    else
        k.cls = 1;
    return k;
}

constexpr int kMaxHRows = 8;   // readout rows per warp held in registers (more: a second pass)

template <typename T, int DPL>
__global__ void __launch_bounds__(DT) decode2_kernel(Dims dm, DevState S, DecodeArgs a, int hpc, void *out_)
{
    constexpr int d = 32 * DPL;
    constexpr int VN = Vec8<T>::N;                   // elements per 16-byte chunk
    constexpr int CPR = d / VN;                      // 16-byte chunks per row
    const int split = blockIdx.x, st = blockIdx.y;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const int D = dm.D, g = dm.g, lam = dm.lam, R = dm.R, nch = dm.dec_nch;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const DecodeSmem L = decode_smem_layout<T, DPL>(D);
    extern __shared__ __align__(16) uint8_t smd[];
    float *qs = (float *)smd;                        // [g][d], scaled by 1/sqrt(d)
    float *phq = (float *)(smd + L.off_phq);         // [g][D]
    int *rowtab = (int *)(smd + L.off_rows) + warp * 2 * 64;   // [2 buffers][row 32 | class 32]
    uint8_t *wbuf = smd + L.off_kv + warp * L.warp_bytes;
    float *red = (float *)(smd + L.off_kv);
    __shared__ int last_cta;
    const float scale = rsqrtf((float)d);

    const long long p = a.pos;
    const long long jlo = a.t0 - dm.eta > 0 ? a.t0 - dm.eta : 0;
    const int nkeys = a.nS + (int)(p - jlo + 1);
    const T *KS = (const T *)S.KS + (size_t)st * lam * d;
    const T *VS = (const T *)S.VS + (size_t)st * lam * d;
    const T *KR = (const T *)S.KR + (size_t)st * R * d;
    const T *VR = (const T *)S.VR + (size_t)st * R * d;
    const T *phiV = (const T *)S.phiV + (size_t)st * (lam + R) * D;

    // this warp's chunks: it = 0..nch-1 -> chunk split*4*nch + warp + 4*it of the stream
    auto chunk_base = [&](int it) { return (split * 4 * nch + warp + 4 * it) * 32; };
    auto stage = [&](int it, int bf) {
        const int kb = chunk_base(it);
        const KeyRef kr = decode_key(dm, S, a, st, kb + lane, nkeys, jlo);
        int *rt = rowtab + bf * 64;
        rt[lane] = kr.row;
        rt[32 + lane] = kr.cls;
        __syncwarp();
        const int nvalid = kb < nkeys ? min(32, nkeys - kb) : 0;
        uint8_t *wk = wbuf + bf * L.buf_bytes, *wv = wk + 32 * L.kstride;
        for (int e = lane; e < nvalid * CPR; e += 32) {
            const int jj = e / CPR, cc = e - jj * CPR;
            const int rw = rt[jj];
            const T *ks = rw < lam ? KS + (size_t)rw * d : KR + (size_t)(rw - lam) * d;
            const T *vs = rw < lam ? VS + (size_t)rw * d : VR + (size_t)(rw - lam) * d;
            cp_async16(wk + jj * L.kstride + cc * 16, ks + cc * VN);
            cp_async16(wv + jj * L.vstride + cc * 16, vs + cc * VN);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    stage(0, 0);

    // queries and their features; the readout rows of this CTA into registers
    const T *qg = (const T *)a.q + ((size_t)b * dm.Hq + (size_t)hk * g) * d;
    const T *pqg = (const T *)S.phiQd + ((size_t)b * dm.Hq + (size_t)hk * g) * D;
    for (int e = tid; e < g * d; e += DT) qs[e] = to_f<T>(qg[e]) * scale;
    for (int e = tid; e < g * D; e += DT) phq[e] = to_f<T>(pqg[e]);
    const float *Hs = S.H + (size_t)st * D * d;
    const float *ss = S.s + (size_t)st * D;
    const int h0 = split * hpc, h1 = min(D, h0 + hpc);
    float hv[kMaxHRows][DPL], hs[kMaxHRows];
#pragma unroll
    for (int k = 0; k < kMaxHRows; ++k) {
        const int i = h0 + warp + 4 * k;
        if (i < h1) {
            load_row<float, DPL>(Hs + (size_t)i * d, lane, hv[k]);
            hs[k] = ss[i];
        } else {
#pragma unroll
            for (int u = 0; u < DPL; ++u) hv[k][u] = 0.f;
            hs[k] = 0.f;
        }
    }
    __syncthreads();

    float m[8], l[8], ld[8], o[8][DPL], lo[8][DPL];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        m[h] = 0.f;          // the shift never goes below 0
        l[h] = 0.f;
        ld[h] = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) o[h][u] = lo[h][u] = 0.f;
    }

    for (int it = 0; it < nch; ++it) {
        const int bf = it & 1;
        if (it + 1 < nch) stage(it + 1, bf ^ 1);
        else asm volatile("cp.async.commit_group;" ::: "memory");   // keep one group in flight
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();
        const int kb = chunk_base(it);
        const int nvalid = kb < nkeys ? min(32, nkeys - kb) : 0;    // warp-uniform
        if (nvalid > 0) {
            const int *rt = rowtab + bf * 64;
            const int row = rt[lane], cls = rt[32 + lane];
            const uint8_t *wk = wbuf + bf * L.buf_bytes, *wv = wk + 32 * L.kstride;
            // scores of this lane's key for every head (key row from shared memory)
            float sc[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) sc[h] = 0.f;
            if (cls == 1) {
                const uint8_t *kr = wk + lane * L.kstride;
#pragma unroll 4
                for (int cc = 0; cc < CPR; ++cc) {
                    float kf[VN];
                    Vec8<T>::load(kr + cc * 16, kf);
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        if (h < g) {
                            const float *qh = qs + h * d + cc * VN;
#pragma unroll
                            for (int u = 0; u < VN; u += 4) {
                                const float4 q4 = *(const float4 *)(qh + u);
                                sc[h] = fmaf(q4.x, kf[u], sc[h]);
                                sc[h] = fmaf(q4.y, kf[u + 1], sc[h]);
                                sc[h] = fmaf(q4.z, kf[u + 2], sc[h]);
                                sc[h] = fmaf(q4.w, kf[u + 3], sc[h]);
                            }
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
            // P V: lane owns value dims [lane*DPL, lane*DPL + DPL); rows from shared memory
            for (int jj = 0; jj < nvalid; ++jj) {
                const T *vr = (const T *)(wv + jj * L.vstride);
                float vf[DPL];
#pragma unroll
                for (int u = 0; u < DPL; ++u) vf[u] = to_f<T>(vr[lane * DPL + u]);
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
        __syncwarp();   // this buffer is refilled two chunks from now
    }
    asm volatile("cp.async.wait_all;" ::: "memory");

    // slice of the readout phi(q)^T H', phi(q)^T s' (unscaled linear sums)
#pragma unroll
    for (int k = 0; k < kMaxHRows; ++k) {
        const int i = h0 + warp + 4 * k;
        if (i < h1) {
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (h < g) {
                    const float f = phq[h * D + i];
#pragma unroll
                    for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(f, hv[k][u], lo[h][u]);
                    ld[h] = fmaf(f, hs[k], ld[h]);
                }
            }
        }
    }
    for (int i = h0 + warp + 4 * kMaxHRows; i < h1; i += 4) {
        float hr[DPL];
        load_row<float, DPL>(Hs + (size_t)i * d, lane, hr);
        const float si = ss[i];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            if (h < g) {
                const float f = phq[h * D + i];
#pragma unroll
                for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(f, hr[u], lo[h][u]);
                ld[h] = fmaf(f, si, ld[h]);
            }
        }
    }
    __syncthreads();   // the staged rows are dead: red[] reuses their space
    // combine the 4 warps, then write this CTA's partial per head
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        if (h < g) {
            float *rw = red + (warp * 8 + h) * (3 + 2 * d);
            if (lane == 0) {
                rw[0] = m[h];
                rw[1] = l[h];
                rw[2] = ld[h];
            }
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                rw[3 + lane * DPL + u] = o[h][u];
                rw[3 + d + lane * DPL + u] = lo[h][u];
            }
        }
    }
    __syncthreads();
    const size_t rec = 2 * d + 4;
    for (int h = warp; h < g; h += 4) {
        float M = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, red[(w * 8 + h) * (3 + 2 * d)]);
        float Ls = 0.f, LD = 0.f, O[DPL], LO[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) O[u] = LO[u] = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float *rw = red + (w * 8 + h) * (3 + 2 * d);
            const float f = __expf(rw[0] - M);
            Ls = fmaf(f, rw[1], Ls);
            LD += rw[2];
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                O[u] = fmaf(f, rw[3 + lane * DPL + u], O[u]);
                LO[u] += rw[3 + d + lane * DPL + u];
            }
        }
        float *pr = S.part + (((size_t)st * dm.nsplit + split) * g + h) * rec;
        if (lane == 0) {
            pr[0] = M;
            pr[1] = Ls;
            pr[2] = LD;
            pr[3] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            pr[4 + lane * DPL + u] = O[u];
            pr[4 + d + lane * DPL + u] = LO[u];
        }
    }

    // the last CTA of the stream merges the splits (online-softmax identity) and writes out
    __threadfence();
    __syncthreads();
    if (tid == 0) last_cta = atomicAdd(&S.dec_cnt[st], 1) == dm.nsplit - 1 ? 1 : 0;
    __syncthreads();
    if (!last_cta) return;
    __threadfence();
    for (int h = warp; h < g; h += 4) {
        const float *base = S.part + ((size_t)st * dm.nsplit * g + h) * rec;
        const size_t sstride = (size_t)g * rec;
        float M = 0.f;
        for (int sp = 0; sp < dm.nsplit; ++sp) M = fmaxf(M, __ldcg(base + sp * sstride));
        float Ls = 0.f, LD = 0.f, O[DPL], LO[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) O[u] = LO[u] = 0.f;
        for (int sp = 0; sp < dm.nsplit; ++sp) {
            const float *pr = base + sp * sstride;
            const float f = __expf(__ldcg(pr) - M);
            Ls = fmaf(f, __ldcg(pr + 1), Ls);
            LD += __ldcg(pr + 2);
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                O[u] = fmaf(f, __ldcg(pr + 4 + lane * DPL + u), O[u]);
                LO[u] += __ldcg(pr + 4 + d + lane * DPL + u);
            }
        }
        const float em = __expf(-M);
        const float rden = 1.f / (Ls + em * (LD + dm.eps));
        T *out = (T *)out_ + ((size_t)b * dm.Hq + (size_t)hk * g + h) * d;
#pragma unroll
        for (int u = 0; u < DPL; ++u) out[lane * DPL + u] = from_f<T>((O[u] + em * LO[u]) * rden);
    }
    if (tid == 0) S.dec_cnt[st] = 0;
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
#define LOLA_DECODE2(T, DPL)                                                                       \
    do {                                                                                           \
        const size_t smem = decode_smem_layout<T, DPL>(dm.D).total;                                \
        cudaFuncSetAttribute(decode2_kernel<T, DPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             (int)smem);                                                           \
        decode2_kernel<T, DPL><<<grid, DT, smem, stream>>>(dm, S, a, hpc, a.out);                  \
    } while (0)
    if (dm.dtype == 0) {
        if (dm.d == 32) LOLA_DECODE2(float, 1);
        else if (dm.d == 64) LOLA_DECODE2(float, 2);
        else LOLA_DECODE2(float, 4);
    } else {
        if (dm.d == 32) LOLA_DECODE2(__nv_bfloat16, 1);
        else if (dm.d == 64) LOLA_DECODE2(__nv_bfloat16, 2);
        else LOLA_DECODE2(__nv_bfloat16, 4);
    }
#undef LOLA_DECODE2
}

void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream)
{
    get_indices_kernel<<<64, 256, 0, stream>>>(dm, S, nS, idx, cnt);
}

}  // namespace lola
