// The sequential part of LoLA's update interval (gist.science technical
// summary, "Inferentiestrategie"), one CTA per (batch, kv-head) stream, walking
// that stream's intervals in order:
//   1. fold the leaving pairs of the previous interval that were not kept
//      (H += phi(k) v^T, s += phi(k));
//   2. score every candidate -- the cached pairs and the pairs leaving the
//      window during this interval -- by the Self-Recall Error
//      SRE(k,v|H,s) = || phi(k)^T H / (phi(k)^T s + eps) - v ||^2
//      ("Het Self-Recall Error (SRE) Mechanisme");
//   3. keep the top min(lambda, |Q|) by SRE, ties to the lower token index;
//   4. fold the evicted cached pairs at once (the state the interval's queries
//      read), then give their slots to the kept leaving pairs.
// Prefill mode records, per interval, the kept set (as token + virtual row),
// the fate of each leaving pair and a snapshot of (H', s') for the attention
// kernel. Decode mode moves kept leaving pairs from the ring into cache slots.
#include "lola_internal.cuh"
#include "scoring.cuh"

namespace lola {

namespace {

constexpr int kFoldTile = 16;
constexpr int kThreads = 512;

// Exclusive block scan of in[0, n) into out[0, n); returns the total.
__device__ int block_exclusive_scan(const int *in, int *out, int n, int *wsum)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int beg = min(n, tid * per), end = min(n, beg + per);
    int local = 0;
    for (int i = beg; i < end; ++i) local += in[i];
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nwarps) wsum[lane] = w;
    }
    __syncthreads();
    int run = (warp > 0 ? wsum[warp - 1] : 0) + x - local;
    for (int i = beg; i < end; ++i) {
        out[i] = run;
        run += in[i];
    }
    const int total = wsum[nwarps - 1];
    __syncthreads();
    return total;
}

// Order-preserving key: ascending key = SRE descending, then token ascending.
__device__ __forceinline__ unsigned long long make_key(float sre, int tok)
{
    const unsigned bits = __float_as_uint(fmaxf(sre, 0.f));
    return ((unsigned long long)(0xFFFFFFFFu - bits) << 32) | (unsigned)tok;
}

// H += sum phi(k_t) v_t^T, s += sum phi(k_t) over the listed virtual rows.
template <typename T>
__device__ void fold_rows(const int *lst, int cnt, const T *__restrict__ phi_st,
                          const KVSrc<T> &src, int st, float *__restrict__ H,
                          float *__restrict__ s, float *stgPhi, float *stgV, int D, int d)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int base = 0; base < cnt; base += kFoldTile) {
        const int nf = min(kFoldTile, cnt - base);
        for (int e = tid; e < nf * D; e += nt) {
            const int t = e / D, i = e - t * D;
            stgPhi[t * D + i] = to_f<T>(phi_st[(size_t)lst[base + t] * D + i]);
        }
        for (int e = tid; e < nf * d; e += nt) {
            const int t = e / d, c = e - t * d;
            stgV[t * d + c] = to_f<T>(src.vrow(st, lst[base + t])[c]);
        }
        __syncthreads();
        for (int e = tid; e < D * d; e += nt) {
            const int i = e / d, c = e - i * d;
            float acc = H[e];
            for (int t = 0; t < nf; ++t) acc = fmaf(stgPhi[t * D + i], stgV[t * d + c], acc);
            H[e] = acc;
        }
        for (int e = tid; e < D; e += nt) {
            float acc = s[e];
            for (int t = 0; t < nf; ++t) acc += stgPhi[t * D + e];
            s[e] = acc;
        }
        __syncthreads();
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    chain_kernel(Dims dm, DevState S, PrefillScratch P, ChainArgs a, KVSrc<T> src)
{
    const int st = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nw = nt >> 5;
    const int D = dm.D, d = dm.d, lam = dm.lam, eta = dm.eta, Lmax = dm.Lmax;
    const int QC = lam + Lmax;

    extern __shared__ __align__(16) unsigned char smraw[];
    unsigned long long *keys = (unsigned long long *)smraw;             // [QC]
    int *ctok = (int *)(keys + QC);                                      // [QC]
    int *cvrow = ctok + QC;                                              // [QC]
    int *keepf = cvrow + QC;                                             // [QC]
    int *tmpA = keepf + QC;                                              // [QC]
    int *tmpB = tmpA + QC;                                               // [QC]
    int *lst = tmpB + QC;                                                // [QC]
    int *slotTok = lst + QC;                                             // [lam]
    int *slotVrow = slotTok + lam;                                       // [lam]
    int *freeSlot = slotVrow + lam;                                      // [lam]
    int *lf = freeSlot + lam;                                            // [Lmax]
    int *scal = lf + Lmax;                                               // [64]
    float *stgPhi = (float *)(scal + 64);                                // [kFoldTile][D]
    float *stgV = stgPhi + kFoldTile * D;                                // [kFoldTile][d]

    float *H = S.H + (size_t)st * D * d;
    float *s = S.s + (size_t)st * D;
    const T *phi_st = (const T *)a.phi + (size_t)st * a.nvrows * D;

    int nS = a.nS0;
    for (int i = tid; i < lam; i += nt) {
        slotTok[i] = i < nS ? S.idxS[(size_t)st * lam + i] : -1;
        slotVrow[i] = i;
    }
    for (int i = tid; i < Lmax; i += nt) lf[i] = i < a.pend_n ? S.pend[(size_t)st * Lmax + i] : 0;
    long long pend_lo = a.pend_lo;
    int pend_n = a.pend_n;
    __syncthreads();

    for (int ci = 0; ci < a.n_int; ++ci) {
        const long long t0 = a.pos0 + (long long)ci * a.ilen;
        const long long t1 = t0 + a.ilen;
        const long long iglob = a.iglob0 + ci;

        // 1. fold the previous interval's leaving pairs that were not kept
        if (pend_n > 0) {
            for (int i = tid; i < pend_n; i += nt) tmpA[i] = lf[i] ? 1 : 0;
            __syncthreads();
            const int nf = block_exclusive_scan(tmpA, tmpB, pend_n, scal);
            for (int i = tid; i < pend_n; i += nt)
                if (tmpA[i]) lst[tmpB[i]] = src.tok2vrow(pend_lo + i);
            __syncthreads();
            fold_rows<T>(lst, nf, phi_st, src, st, H, s, stgPhi, stgV, D, d);
        }

        // 2. candidates: cache slots, then pairs leaving the window in [t0, t1)
        const long long Llo = t0 - eta > 0 ? t0 - eta : 0;
        const long long Lhi = t1 - eta > Llo ? t1 - eta : Llo;
        const int nL = (int)(Lhi - Llo);
        const int nQ = nS + nL;
        for (int c = tid; c < nQ; c += nt) {
            if (c < nS) {
                ctok[c] = slotTok[c];
                cvrow[c] = slotVrow[c];
            } else {
                const long long tok = Llo + (c - nS);
                ctok[c] = (int)tok;
                cvrow[c] = src.tok2vrow(tok);
            }
        }
        __syncthreads();

        //    Self-Recall Error against the state at the interval start (or an ablation score)
        const int nDu = D >> 5, ndu = d >> 5;
        if (dm.scorer != kScoreSRE) {
            float *score = (float *)keepf, *lg = (float *)tmpA, *lu = (float *)tmpB;
            float *qs = stgPhi, *pq = stgPhi + dm.g * d, *red = (float *)scal;
            const T *qb = (const T *)a.qin;
            const int b = st / dm.Hkv, hk = st % dm.Hkv;
            const size_t qrow0 = (((size_t)b * a.q_n + (size_t)(t0 - a.q_start)) * dm.Hq + (size_t)hk * dm.g) * d;
            alt_scores<T>(
                dm.scorer, nQ, [&](int c) { return src.krow(st, cvrow[c]); },
                [&](int c) { return phi_st + (size_t)cvrow[c] * D; }, [&](int h) { return qb + qrow0 + (size_t)h * d; },
                [&](int c) { return ctok[c]; }, w_of(dm, S.W, hk), dm.g, d, D, score, qs, pq, lg, lu, red);
            for (int c = tid; c < nQ; c += nt) {
                keys[c] = make_key(score[c], ctok[c]);
                if (a.score_sre != nullptr && iglob < a.score_cap) {
                    const size_t o = ((size_t)iglob * dm.ns + st) * QC + c;
                    a.score_sre[o] = score[c];
                    a.score_tok[o] = ctok[c];
                }
            }
        }
        for (int c = dm.scorer == kScoreSRE ? warp : nQ; c < nQ; c += nw) {
            const T *ph = phi_st + (size_t)cvrow[c] * D;
            float phr[8];
            float den = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (u < nDu) {
                    phr[u] = to_f<T>(ph[lane + 32 * u]);
                    den = fmaf(phr[u], s[lane + 32 * u], den);
                } else {
                    phr[u] = 0.f;
                }
            }
            den = warp_sum(den) + dm.eps;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (u < nDu) {
                    for (int l = 0; l < 32; ++l) {
                        const float f = __shfl_sync(0xffffffffu, phr[u], l);
                        const float *hr = H + (size_t)(32 * u + l) * d;
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            if (w < ndu) acc[w] = fmaf(f, hr[lane + 32 * w], acc[w]);
                    }
                }
            }
            const T *vr = src.vrow(st, cvrow[c]);
            float e = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                if (w < ndu) {
                    const float pred = den != 0.f ? acc[w] / den : 0.f;
                    const float diff = pred - to_f<T>(vr[lane + 32 * w]);
                    e = fmaf(diff, diff, e);
                }
            }
            e = warp_sum(e);
            if (lane == 0) {
                keys[c] = make_key(e, ctok[c]);
                if (a.score_sre != nullptr && iglob < a.score_cap) {
                    const size_t o = ((size_t)iglob * dm.ns + st) * QC + c;
                    a.score_sre[o] = e;
                    a.score_tok[o] = ctok[c];
                }
            }
        }
        __syncthreads();

        // 3. top min(lam, |Q|): rank of each key among all keys (keys are unique)
        const int nK = nQ < lam ? nQ : lam;
        for (int c = tid; c < nQ; c += nt) {
            const unsigned long long kc = keys[c];
            int r = 0;
            for (int c2 = 0; c2 < nQ; ++c2) r += keys[c2] < kc ? 1 : 0;
            keepf[c] = r < nK ? 1 : 0;
        }
        __syncthreads();
        if (a.sel_log != nullptr && iglob < a.sel_cap) {
            int32_t *lg = a.sel_log + ((size_t)iglob * dm.ns + st) * (lam + 1);
            const int cnt = block_exclusive_scan(keepf, tmpB, nQ, scal);
            for (int c = tid; c < nQ; c += nt)
                if (keepf[c]) lg[1 + tmpB[c]] = ctok[c];
            for (int i = cnt + tid; i < lam; i += nt) lg[1 + i] = -1;
            if (tid == 0) lg[0] = cnt;
        }
        const int32_t *lst_o =
            (a.ovr != nullptr && iglob < a.ovr_n) ? a.ovr + ((size_t)iglob * dm.ns + st) * (lam + 1)
                                                  : nullptr;
        if (lst_o != nullptr && lst_o[0] >= 0) {   // a negative count leaves this entry unforced
            const int cnt = lst_o[0];
            if (tid == 0 && cnt != nK) raise_error(S.err, ERR_BOUNDS);
            for (int c = tid; c < nQ; c += nt) {
                int lo = 0, hi = cnt < lam ? cnt : lam;
                const int key = ctok[c];
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (lst_o[1 + mid] < key) lo = mid + 1; else hi = mid;
                }
                keepf[c] = (lo < cnt && lo < lam && lst_o[1 + lo] == key) ? 1 : 0;
            }
            __syncthreads();
        }

        // 4a. evicted cached pairs E = S n F: fold now (H' for this interval's queries)
        for (int c = tid; c < nS; c += nt) tmpA[c] = keepf[c] ? 0 : 1;
        __syncthreads();
        const int nE = block_exclusive_scan(tmpA, tmpB, nS, scal);
        for (int c = tid; c < nS; c += nt) {
            if (tmpA[c]) {
                lst[tmpB[c]] = cvrow[c];
                freeSlot[tmpB[c]] = c;
            }
        }
        for (int r = nE + tid; r < nE + (lam - nS); r += nt) freeSlot[r] = nS + (r - nE);
        __syncthreads();
        fold_rows<T>(lst, nE, phi_st, src, st, H, s, stgPhi, stgV, D, d);
        if (a.mode == 0) {
            float *sh = P.snapH + ((size_t)st * dm.mmax + ci) * D * d;
            float *ss = P.snapS + ((size_t)st * dm.mmax + ci) * D;
            for (int e = tid; e < D * d; e += nt) sh[e] = H[e];
            for (int e = tid; e < D; e += nt) ss[e] = s[e];
        }

        // 4b. kept leaving pairs take the free slots (E slots first, ascending)
        for (int c = tid; c < nL; c += nt) tmpA[c] = keepf[nS + c];
        __syncthreads();
        const int nNew = block_exclusive_scan(tmpA, tmpB, nL, scal);
        if (tid == 0 && nNew > nE + (lam - nS)) raise_error(S.err, ERR_BOUNDS);
        for (int c = tid; c < nL; c += nt) {
            if (tmpA[c] && tmpB[c] < nE + (lam - nS)) {
                const int slot = freeSlot[tmpB[c]];
                slotTok[slot] = ctok[nS + c];
                slotVrow[slot] = a.mode == 0 ? cvrow[nS + c] : slot;
            }
        }
        if (a.mode == 1) {
            // move the new members' rows from the ring into their cache slots
            T *KS = (T *)S.KS + (size_t)st * lam * d;
            T *VS = (T *)S.VS + (size_t)st * lam * d;
            T *phiV = (T *)S.phiV + (size_t)st * a.nvrows * D;
            for (int c = warp; c < nL; c += nw) {
                if (!tmpA[c] || tmpB[c] >= nE + (lam - nS)) continue;
                const int slot = freeSlot[tmpB[c]];
                const int vr = cvrow[nS + c];
                const T *kr = src.krow(st, vr);
                const T *vv = src.vrow(st, vr);
                for (int e = lane; e < d; e += 32) {
                    KS[(size_t)slot * d + e] = kr[e];
                    VS[(size_t)slot * d + e] = vv[e];
                }
                for (int e = lane; e < D; e += 32)
                    phiV[(size_t)slot * D + e] = phiV[(size_t)vr * D + e];
                if (lane == 0) S.idxS[(size_t)st * lam + slot] = ctok[nS + c];
            }
        }
        __syncthreads();

        if (a.mode == 0) {
            const size_t lb = (size_t)st * dm.mmax + ci;
            for (int i = tid; i < nK; i += nt) {
                P.logTok[lb * lam + i] = slotTok[i];
                P.logVrow[lb * lam + i] = slotVrow[i];
            }
            for (int c = tid; c < nL; c += nt) {
                const long long j = Llo + c;
                P.logLf[lb * Lmax + (int)(j - (t0 - eta))] = keepf[nS + c] ? 0 : 1;
            }
            if (tid == 0) P.logCount[lb] = nK;
        }
        // leaving pairs that were not kept become the next interval's pending fold
        for (int c = tid; c < nL; c += nt) lf[c] = keepf[nS + c] ? 0 : 1;
        pend_lo = Llo;
        pend_n = nL;
        nS = nK;
        __syncthreads();
    }

    for (int i = tid; i < Lmax; i += nt) S.pend[(size_t)st * Lmax + i] = (uint8_t)(i < pend_n ? lf[i] : 0);
    if (a.mode == 0) {
        for (int i = tid; i < lam; i += nt) {
            P.slotTok[(size_t)st * lam + i] = slotTok[i];
            P.slotVrow[(size_t)st * lam + i] = slotVrow[i];
        }
    }
}

size_t chain_smem(const Dims &dm)
{
    const size_t QC = (size_t)dm.lam + dm.Lmax;
    return QC * 8 + QC * 4 * 6 + (size_t)dm.lam * 4 * 3 + (size_t)dm.Lmax * 4 + 64 * 4 +
           (size_t)kFoldTile * (dm.D + dm.d) * 4;
}

template <typename T>
void launch_chain_t(const Dims &dm, const DevState &S, const PrefillScratch *P, const ChainArgs &a,
                    cudaStream_t stream)
{
    KVSrc<T> src{(const T *)S.KS, (const T *)S.VS, (const T *)S.KR, (const T *)S.VR,
                 (const T *)a.kin, (const T *)a.vin, dm.lam, dm.R, a.n_call, dm.Hkv, dm.d,
                 a.call_start};
    const size_t smem = chain_smem(dm);
    cudaFuncSetAttribute(chain_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    PrefillScratch Pv{};
    if (P) Pv = *P;
    chain_kernel<T><<<dm.ns, kThreads, smem, stream>>>(dm, S, Pv, a, src);
}

}  // namespace

void launch_chain(const Dims &dm, const DevState &S, const PrefillScratch *P, const ChainArgs &a,
                  cudaStream_t stream)
{
    if (dm.dtype == 0)
        launch_chain_t<float>(dm, S, P, a, stream);
    else
        launch_chain_t<__nv_bfloat16>(dm, S, P, a, stream);
}

size_t chain_smem_bytes(const Dims &dm) { return chain_smem(dm); }

}  // namespace lola
