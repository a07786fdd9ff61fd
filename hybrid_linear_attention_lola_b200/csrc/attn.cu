// Prefill output of a LoLA hybrid-attention layer (gist.science technical
// summary, "Inferentiestrategie", last step: the output combines the linear
// attention, the sparse-cache attention and the sliding-window attention).
//
// For query p of interval [t0, t1) and key j <= p:
//   softmax weight e^{q.k/sqrt(d)}  if j is in the interval's kept set, or j is
//                                   inside the window of p (j > p - eta);
//   linear weight  phi(q).phi(k_j)  if j left the window during the interval
//                                   (j <= p - eta) and was folded;
// plus the readout phi(q)^T H', phi(q)^T s' of the state after the interval's
// cache evictions. All terms share one normaliser (+ eps); the softmax terms are
// evaluated with the running shift m = max(0, max score) and the linear terms
// carry e^{-m}, which merges partial numerators/denominators in any order (the
// online-softmax identity).
//
// One CTA = 64 query rows of one query head in one interval; one warp = 8 rows.
#include "lola_internal.cuh"

namespace lola {

namespace {

constexpr int QR = 64;   // query rows per CTA
constexpr int KT = 32;   // keys per tile
constexpr int NW = 8;    // warps per CTA
constexpr int RPW = QR / NW;

enum : int { CLS_NONE = 0, CLS_SOFT = 1, CLS_LIN = 2 };
enum : int { KINFO_WINDOW = 0, KINFO_FOLDED = 1, KINFO_SKIP = 2 };

struct RowAcc {
    float m, l, ld;
    float nsm[4], nln[4];
};

template <typename T>
__global__ void __launch_bounds__(NW * 32)
    attn_prefill_kernel(Dims dm, PrefillScratch P, AttnArgs a, KVSrc<T> src, const int *err)
{
    if (cta_error_pending(err)) return;   // the chain of this call gave up: its logs are incomplete
    const int d = dm.d, D = dm.D, eta = dm.eta, lam = dm.lam;
    const int qsplit = (dm.C + QR - 1) / QR;
    const int ci = a.ci0 + blockIdx.x / qsplit, qp = blockIdx.x % qsplit;
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hk = hq / dm.g, st = b * dm.Hkv + hk;
    const long long t0 = a.pos0 + (long long)ci * dm.C, t1 = t0 + dm.C;
    const int row0 = qp * QR;
    const int nrows = min(QR, dm.C - row0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ndu = d >> 5;
    const float scale = rsqrtf((float)d);

    extern __shared__ __align__(16) float sm[];
    float *qs = sm;                          // [QR][d]
    float *phq = qs + QR * d;                // [QR][D]
    float *Ks = phq + QR * D;                // [KT][d + 1]
    float *Vs = Ks + KT * (d + 1);           // [KT][d]
    float *phk = Vs + KT * d;                // [KT][D + 1]
    int *ktok = (int *)(phk + KT * (D + 1)); // [KT]
    int *kinfo = ktok + KT;                  // [KT]
    int *flag = kinfo + KT;                  // [4]

    const T *q = (const T *)a.q;
    for (int e = tid; e < nrows * d; e += blockDim.x) {
        const int r = e / d, c = e - r * d;
        const long long tok = t0 - a.pos0 + row0 + r;
        qs[e] = to_f<T>(q[(((size_t)b * a.n_call + tok) * dm.Hq + hq) * d + c]) * scale;
    }
    for (int e = tid; e < nrows * D; e += blockDim.x) {
        const int r = e / D, i = e - r * D;
        const long long tok = t0 - a.pos0 + row0 + r;
        phq[e] = to_f<T>(((const T *)P.phiQ)[(((size_t)b * a.n_call + tok) * dm.Hq + hq) * D + i]);
    }

    RowAcc acc[RPW];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        acc[rr].m = 0.f;
        acc[rr].l = 0.f;
        acc[rr].ld = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[rr].nsm[w] = acc[rr].nln[w] = 0.f;
    }

    const size_t lb = (size_t)st * dm.mmax + ci;
    const int nK = P.logCount[lb];
    const int *ltok = P.logTok + lb * lam;
    const int *lvrow = P.logVrow + lb * lam;
    const uint8_t *llf = P.logLf + lb * dm.Lmax;
    const long long jlo = t0 - eta > 0 ? t0 - eta : 0;
    const long long nband = t1 - jlo;
    const long long ntiles_c = (nK + KT - 1) / KT;
    const long long ntiles = ntiles_c + (nband + KT - 1) / KT;

    for (long long tile = 0; tile < ntiles; ++tile) {
        const bool band = tile >= ntiles_c;
        const long long kb = band ? jlo + (tile - ntiles_c) * KT : tile * KT;
        const int nk = band ? (int)min((long long)KT, t1 - kb) : (int)min((long long)KT, (long long)nK - kb);
        __syncthreads();
        if (tid < 4) flag[tid] = 0;
        __syncthreads();
        if (tid < KT) {
            int tok = -1, info = KINFO_SKIP;
            if (tid < nk) {
                if (band) {
                    const long long j = kb + tid;
                    tok = (int)j;
                    if (j < t1 - eta) {
                        const int folded = llf[(int)(j - (t0 - eta))];
                        info = folded ? KINFO_FOLDED : KINFO_SKIP;
                    } else {
                        info = KINFO_WINDOW;
                    }
                    if (info == KINFO_FOLDED) flag[0] = 1;
                } else {
                    tok = ltok[kb + tid];
                    info = KINFO_WINDOW;  // cached: softmax whenever causal
                }
            }
            ktok[tid] = tok;
            kinfo[tid] = info;
        }
        __syncthreads();
        const bool any_lin = flag[0] != 0;
        for (int e = tid; e < nk * d; e += blockDim.x) {
            const int j = e / d, c = e - j * d;
            const int vr = band ? src.tok2vrow(kb + j) : lvrow[kb + j];
            Ks[j * (d + 1) + c] = to_f<T>(src.krow(st, vr)[c]);
            Vs[j * d + c] = to_f<T>(src.vrow(st, vr)[c]);
        }
        if (any_lin) {
            for (int e = tid; e < nk * D; e += blockDim.x) {
                const int j = e / D, i = e - j * D;
                const int vr = src.tok2vrow(kb + j);
                phk[j * (D + 1) + i] =
                    to_f<T>(((const T *)P.phiK)[((size_t)st * (lam + dm.R + dm.Nmax) + vr) * D + i]);
            }
        }
        __syncthreads();

        const int mytok = lane < nk ? ktok[lane] : -1;
        const int myinfo = lane < nk ? kinfo[lane] : KINFO_SKIP;
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const int row = warp * RPW + rr;
            if (row >= nrows) continue;  // warp-uniform
            const long long p = t0 + row0 + row;
            int cls = CLS_NONE;
            if (lane < nk && myinfo != KINFO_SKIP && mytok <= p) {
                cls = (myinfo == KINFO_FOLDED && mytok <= p - eta) ? CLS_LIN : CLS_SOFT;
            }
            float sc = -INFINITY;
            if (cls == CLS_SOFT) {
                const float *qr = qs + row * d;
                const float *kr = Ks + lane * (d + 1);
                float dot = 0.f;
                for (int c = 0; c < d; ++c) dot = fmaf(qr[c], kr[c], dot);
                sc = dot;
            }
            const float tmax = warp_max(sc);
            RowAcc &A = acc[rr];
            if (tmax > A.m) {
                const float f = __expf(A.m - tmax);
                A.l *= f;
#pragma unroll
                for (int w = 0; w < 4; ++w) A.nsm[w] *= f;
                A.m = tmax;
            }
            const float pw = cls == CLS_SOFT ? __expf(sc - A.m) : 0.f;
            A.l += warp_sum(pw);
            float lw = 0.f;
            if (any_lin) {
                if (cls == CLS_LIN) {
                    const float *pq = phq + row * D;
                    const float *pk = phk + lane * (D + 1);
                    float dot = 0.f;
                    for (int i = 0; i < D; ++i) dot = fmaf(pq[i], pk[i], dot);
                    lw = dot;
                }
                A.ld += warp_sum(lw);
            }
            for (int jj = 0; jj < nk; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, pw, jj);
                const float lj = __shfl_sync(0xffffffffu, lw, jj);
                const float *vr = Vs + jj * d;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (w < ndu) {
                        const float vv = vr[lane + 32 * w];
                        A.nsm[w] = fmaf(pj, vv, A.nsm[w]);
                        A.nln[w] = fmaf(lj, vv, A.nln[w]);
                    }
                }
            }
        }
    }

    // readout of (H', s') after the interval's evictions, 32 feature rows at a time
    const float *sh = P.snapH + lb * D * d;
    const float *ss = P.snapS + lb * D;
    float *Hs = Vs;      // reuse: [KT][d]
    float *sS = phk;     // reuse: [KT]
    for (int i0 = 0; i0 < D; i0 += KT) {
        __syncthreads();
        for (int e = tid; e < KT * d; e += blockDim.x) Hs[e] = sh[(size_t)i0 * d + e];
        if (tid < KT) sS[tid] = ss[i0 + tid];
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const int row = warp * RPW + rr;
            if (row >= nrows) continue;
            RowAcc &A = acc[rr];
            const float *pq = phq + row * D + i0;
            float dd = 0.f;
            for (int ii = 0; ii < KT; ++ii) {
                const float f = pq[ii];
                dd = fmaf(f, sS[ii], dd);
                const float *hr = Hs + ii * d;
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    if (w < ndu) A.nln[w] = fmaf(f, hr[lane + 32 * w], A.nln[w]);
            }
            A.ld += dd;
        }
    }

    T *out = (T *)a.out;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        const int row = warp * RPW + rr;
        if (row >= nrows) continue;
        const RowAcc &A = acc[rr];
        const float em = __expf(-A.m);
        const float den = A.l + em * (A.ld + dm.eps);
        const long long tok = t0 - a.pos0 + row0 + row;
        T *o = out + (((size_t)b * a.n_call + tok) * dm.Hq + hq) * d;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            if (w < ndu) o[lane + 32 * w] = from_f<T>((A.nsm[w] + em * A.nln[w]) / den);
    }
}

size_t attn_smem(const Dims &dm)
{
    return sizeof(float) * ((size_t)QR * dm.d + (size_t)QR * dm.D + (size_t)KT * (dm.d + 1) +
                            (size_t)KT * dm.d + (size_t)KT * (dm.D + 1)) +
           sizeof(int) * (2 * KT + 4);
}

// ---------------------------------------------------------------- finalize

// One copy unit of a key/value row: 16 bytes when the row is a whole number of them.
template <typename T> __device__ __forceinline__ int row_vec(int d)
{
    return (d * (int)sizeof(T)) % 16 == 0 ? 16 / (int)sizeof(T) : 1;
}
template <typename T> __device__ __forceinline__ void copy_unit(T *dst, const T *src, int vec)
{
    if (vec * sizeof(T) == 16) *(uint4 *)dst = *(const uint4 *)src;
    else for (int k = 0; k < vec; ++k) dst[k] = src[k];
}

// Cache slot i <- its pair's key/value row (from the window ring or this call's input),
// idxS <- its token; one thread per (stream, slot, copy unit) over the whole grid.
template <typename T>
__global__ void finalize_cache_kernel(Dims dm, DevState S, PrefillScratch P, KVSrc<T> src, int nK)
{
    if (*(const volatile int *)S.err != 0) return;   // the chain gave up: slot rows may be incomplete
    const int lam = dm.lam, d = dm.d;
    const int vec = row_vec<T>(d), upr = d / vec;
    const long long total = (long long)dm.ns * lam * upr;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int u = (int)(e % upr);
        const long long rs = e / upr;
        const int i = (int)(rs % lam), st = (int)(rs / lam);
        const size_t slot = (size_t)st * lam + i;
        if (i >= nK) {
            if (u == 0) S.idxS[slot] = -1;
            continue;
        }
        const int vr = P.slotVrow[slot];
        if (vr >= lam) {
            copy_unit((T *)S.KS + slot * d + u * vec, src.krow(st, vr) + u * vec, vec);
            copy_unit((T *)S.VS + slot * d + u * vec, src.vrow(st, vr) + u * vec, vec);
        } else if (vr != i && u == 0) {
            raise_error(S.err, ERR_BOUNDS);
        }
        if (u == 0) S.idxS[slot] = P.slotTok[slot];
    }
}

// Ring slot (token mod R) <- the call's last min(n, R) tokens; one thread per copy unit.
template <typename T>
__global__ void ring_update_kernel(Dims dm, DevState S, const T *__restrict__ kin,
                                   const T *__restrict__ vin, long long call_start, int n)
{
    const int first = n > dm.R ? n - dm.R : 0;
    const int cnt = n - first;
    const int vec = row_vec<T>(dm.d), upr = dm.d / vec;
    const long long total = (long long)cnt * dm.ns * upr;
    T *KR = (T *)S.KR, *VR = (T *)S.VR;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int u = (int)(e % upr);
        const long long r = e / upr;
        const int st = (int)(r % dm.ns);
        const int t = first + (int)(r / dm.ns);
        const int b = st / dm.Hkv, hk = st % dm.Hkv;
        const long long tok = call_start + t;
        const int slot = (int)(tok & (dm.R - 1));
        const size_t so = (((size_t)b * n + t) * dm.Hkv + hk) * dm.d + (size_t)u * vec;
        const size_t dof = ((size_t)st * dm.R + slot) * dm.d + (size_t)u * vec;
        copy_unit(KR + dof, kin + so, vec);
        copy_unit(VR + dof, vin + so, vec);
    }
}

template <typename T>
KVSrc<T> make_src(const Dims &dm, const DevState &S, const void *kin, const void *vin,
                  long long call_start, int n)
{
    return KVSrc<T>{(const T *)S.KS, (const T *)S.VS, (const T *)S.KR, (const T *)S.VR,
                    (const T *)kin, (const T *)vin, dm.lam, dm.R, n, dm.Hkv, dm.d, call_start};
}

}  // namespace

void launch_attn_prefill(const Dims &dm, const DevState &S, const PrefillScratch &P,
                         const AttnArgs &a, cudaStream_t stream)
{
    const int qsplit = (dm.C + QR - 1) / QR;
    dim3 grid(a.m * qsplit, dm.Hq, dm.B);
    const size_t smem = attn_smem(dm);
    if (dm.dtype == 0) {
        cudaFuncSetAttribute(attn_prefill_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        attn_prefill_kernel<float><<<grid, NW * 32, smem, stream>>>(
            dm, P, a, make_src<float>(dm, S, a.kin, a.vin, a.pos0, a.n_call), S.err);
    } else {
        cudaFuncSetAttribute(attn_prefill_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        attn_prefill_kernel<__nv_bfloat16><<<grid, NW * 32, smem, stream>>>(
            dm, P, a, make_src<__nv_bfloat16>(dm, S, a.kin, a.vin, a.pos0, a.n_call), S.err);
    }
}

void launch_finalize_prefill(const Dims &dm, const DevState &S, const PrefillScratch &P,
                             const void *kin, const void *vin, long long call_start, int n,
                             int nK, cudaStream_t stream)
{
    auto blocks = [](long long units) {
        long long g = (units + 255) / 256;
        if (g > 148 * 8) g = 148 * 8;
        return (int)(g < 1 ? 1 : g);
    };
    // upper bounds of the copy units (one per element when rows are not whole 16-byte units)
    const long long ring_units = (long long)(n > dm.R ? dm.R : n) * dm.ns * dm.d;
    const long long cache_units = (long long)dm.ns * dm.lam * dm.d;
    const int g = blocks(ring_units / 4 + 1), gc = blocks(cache_units / 4 + 1);
    if (dm.dtype == 0) {
        finalize_cache_kernel<float><<<gc, 256, 0, stream>>>(
            dm, S, P, make_src<float>(dm, S, kin, vin, call_start, n), nK);
        ring_update_kernel<float><<<g, 256, 0, stream>>>(dm, S, (const float *)kin,
                                                              (const float *)vin, call_start, n);
    } else {
        finalize_cache_kernel<__nv_bfloat16><<<gc, 256, 0, stream>>>(
            dm, S, P, make_src<__nv_bfloat16>(dm, S, kin, vin, call_start, n), nK);
        ring_update_kernel<__nv_bfloat16><<<g, 256, 0, stream>>>(
            dm, S, (const __nv_bfloat16 *)kin, (const __nv_bfloat16 *)vin, call_start, n);
    }
}

size_t attn_smem_bytes(const Dims &dm) { return attn_smem(dm); }

}  // namespace lola
