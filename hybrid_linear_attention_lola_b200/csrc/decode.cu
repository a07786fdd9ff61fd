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
//
// One kernel per step streams everything a step reads exactly once from HBM.
// A stream's work is cut into items of 32 rows: key chunks (32 keys: their key
// and value rows) and state chunks (32 feature rows of H and s). The items are
// dealt round-robin to the warps of the stream's CTAs; every warp copies its
// next items into a ring of shared-memory buffers with bulk asynchronous copies
// (TMA, one mbarrier per buffer) while it works on the current one. Scores:
// one lane per key against the g queries of the group (shared memory). P V:
// one lane per pair of value dimensions, the key weights broadcast from shared
// memory. The online-softmax state of every warp is merged at the end, across
// the CTAs of a stream by the last CTA to finish (a per-stream counter).
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {

namespace {

constexpr int kMaxG = 8;
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s per staging-buffer wait
constexpr int kSMs = 148;

// ---------------------------------------------------------------- shared memory plan

struct DecLayout {
    size_t off_xs, off_qs, off_z, off_phq, off_pw, off_pend, off_mb, total;
    int qs_stride;   // floats per padded, scaled query row
    int ps_stride;   // floats per padded phi(q) row
};

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) / 16 * 16; }

// [staging ring: nw x nst x sb][raw rows: 9 x d][scaled queries: 8 padded rows]
// [z: 9 x Dh][phi(q): 8 padded rows][key weights: nw x 8 x 32][fates: Lmax]
// [mbarriers: nw x nst]; the final merge reuses the ring.
__host__ __device__ inline DecLayout dec_layout(const Dims &dm)
{
    DecLayout L{};
    const int d = dm.d;
    L.qs_stride = d + d / 8;
    L.ps_stride = dm.D + dm.D / 8;
    size_t o = (size_t)dm.dec_nw * dm.dec_nst * dm.dec_sb;
    L.off_xs = o;
    o = al16(o + (size_t)(kMaxG + 1) * d * 4);
    L.off_qs = o;
    o = al16(o + (size_t)kMaxG * L.qs_stride * 4);
    L.off_z = o;
    o = al16(o + (size_t)(kMaxG + 1) * dm.Dh * 4);
    L.off_phq = o;
    o = al16(o + (size_t)kMaxG * L.ps_stride * 4);
    L.off_pw = o;
    o = al16(o + (size_t)dm.dec_nw * kMaxG * 32 * 4);
    L.off_pend = o;
    o = al16(o + (size_t)dm.Lmax);
    L.off_mb = o;
    o += (size_t)dm.dec_nw * dm.dec_nst * 8;
    L.total = o;
    return L;
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16 bytes of T as floats
template <typename T> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const uint8_t *p, float *f)
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
template <> struct Chunk<float> {
    static constexpr int N = 4;
    __device__ static void load(const uint8_t *p, float *f)
    {
        const float4 r = *(const float4 *)p;
        f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
    }
};

// Offset (floats) of element i of 16-byte chunk c of a padded row (queries,
// features): with 8-float chunks, chunks 4..7 of every 8 are shifted by 4
// floats so that the 8 lanes of a 128-bit shared-memory phase, which read 8
// distinct chunks of a group of 8, hit distinct banks.
template <int VN> __device__ __forceinline__ int qoff(int c, int i)
{
    return VN == 8 ? c * 8 + ((c >> 2) & 1) * 4 + (c >> 3) * 8 + i : c * VN + i;
}
template <int VN> __device__ __forceinline__ int qidx(int x) { return qoff<VN>(x / VN, x % VN); }

// Work items of one stream for the step at position p (identical in every CTA):
//   [0, nkc)            32 softmax keys: cache slots [0, nS), then window tokens [wlo, p]
//   [nkc, nkc + nlc)    16 linear-band tokens of [jlo, lhi) (left the window this
//                       interval; folded ones are linear, kept ones are skipped)
//   [nkc + nlc, ni)     32 feature rows of the state (H, s)
struct Items {
    long long jlo, wlo, lhi;
    int nsoft, nkc, nlc, ni;
};

__device__ __forceinline__ Items make_items(const Dims &dm, const DecodeArgs &a)
{
    Items it;
    const long long p = a.pos;
    it.jlo = a.t0 - dm.eta > 0 ? a.t0 - dm.eta : 0;
    it.wlo = p - dm.eta + 1 > it.jlo ? p - dm.eta + 1 : it.jlo;
    it.lhi = a.L_hi < it.wlo ? a.L_hi : it.wlo;
    if (it.lhi < it.jlo) it.lhi = it.jlo;
    it.nsoft = a.nS + (int)(p - it.wlo + 1);
    it.nkc = (it.nsoft + 31) / 32;
    it.nlc = (int)((it.lhi - it.jlo + 15) / 16);
    it.ni = it.nkc + it.nlc + dm.D / 32;
    return it;
}

template <typename T, int DPL>
__global__ void __launch_bounds__(128) decode3_kernel(Dims dm, DevState S, DecodeArgs a, int do_append)
{
    constexpr int d = 32 * DPL;
    constexpr int E = (int)sizeof(T);
    constexpr int VN = Chunk<T>::N;
    constexpr int CPR = d / VN;                        // 16-byte chunks per key row
    constexpr int XM = CPR >= 8 ? 7 : CPR - 1;         // chunk-order rotation mask
    const int nw = dm.dec_nw, nst = dm.dec_nst, SB = dm.dec_sb;
    const int split = blockIdx.x, st = blockIdx.y;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
    const int D = dm.D, Dh = dm.Dh, g = dm.g, lam = dm.lam, R = dm.R;
    const long long p = a.pos;
    const int nS = a.nS;
    const Items IT = make_items(dm, a);
    const int gw = split * nw + warp, wstride = dm.nsplit * nw;
    const int nmine = gw < IT.ni ? (IT.ni - gw + wstride - 1) / wstride : 0;
    const DecLayout L = dec_layout(dm);
    const int QS = L.qs_stride, PS = L.ps_stride;
    const int CPD = D / VN;                            // 16-byte chunks per phi row
    const int XMD = CPD >= 16 ? 7 : (CPD >> 1) - 1;    // rotation within half a phi row

    extern __shared__ __align__(128) uint8_t smd[];
    uint8_t *ring = smd + (size_t)warp * nst * SB;
    float *xs = (float *)(smd + L.off_xs);   // raw rows: the g queries, then the new key
    float *qs = (float *)(smd + L.off_qs);   // queries scaled by 1/sqrt(d), padded layout
    float *zs = (float *)(smd + L.off_z);
    float *phq = (float *)(smd + L.off_phq); // phi(q), padded layout
    float *pws = (float *)(smd + L.off_pw) + warp * kMaxG * 32;
    uint8_t *fate = smd + L.off_pend;        // 1 = leaving pair of this interval that is folded
    uint64_t *mb = (uint64_t *)(smd + L.off_mb) + warp * nst;
    __shared__ int last_cta;

    const T *KS = (const T *)S.KS + (size_t)st * lam * d;
    const T *VS = (const T *)S.VS + (size_t)st * lam * d;
    const T *KR = (const T *)S.KR + (size_t)st * R * d;
    const T *VR = (const T *)S.VR + (size_t)st * R * d;
    const T *kin = (const T *)a.k + (size_t)st * d;
    const T *vin = (const T *)a.v + (size_t)st * d;
    const float *Hg = S.H + (size_t)st * D * d;
    const float *sg = S.s + (size_t)st * D;
    T *phiV = (T *)S.phiV + (size_t)st * (lam + R) * D;

    if (lane == 0)
        for (int i = 0; i < nst; ++i) umma::mbar_init(&mb[i], 1);
    __syncwarp();

    // copies ring rows of tokens [j, j + n) (no token p among them) to dst (lane 0)
    auto ring_rows = [&](uint8_t *dst, const T *base_, long long j, int n, uint32_t rb, int stride,
                         uint64_t *bar) {
        while (n > 0) {
            const int slot = (int)(j & (R - 1));
            const int m = min(n, R - slot);
            umma::bulk_g2s(dst, base_ + (size_t)slot * stride, (uint32_t)m * rb, bar);
            dst += (size_t)m * rb;
            j += m;
            n -= m;
        }
    };
    // copies item k of this warp into buffer s (lane 0)
    auto issue = [&](int k, int s) {
        const int it = gw + k * wstride;
        uint8_t *buf = ring + (size_t)s * SB;
        uint64_t *bar = &mb[s];
        const uint32_t rb = (uint32_t)(d * E);
        if (it < IT.nkc) {
            const int k0 = it * 32, k1 = min(k0 + 32, IT.nsoft);
            umma::mbar_arrive_expect_tx(bar, (uint32_t)(k1 - k0) * rb * 2);
            uint8_t *kd = buf, *vd = buf + 32 * rb;
            int key = k0;
            if (key < nS) {
                const int c1 = min(k1, nS);
                umma::bulk_g2s(kd, KS + (size_t)key * d, (uint32_t)(c1 - key) * rb, bar);
                umma::bulk_g2s(vd, VS + (size_t)key * d, (uint32_t)(c1 - key) * rb, bar);
                key = c1;
            }
            if (key < k1) {
                const long long j = IT.wlo + (key - nS);
                const int off = key - k0;
                const long long jend = IT.wlo + (k1 - nS);        // exclusive
                const int nring = (int)((jend < p ? jend : p) - j);
                if (nring > 0) {
                    ring_rows(kd + (size_t)off * rb, KR, j, nring, rb, d, bar);
                    ring_rows(vd + (size_t)off * rb, VR, j, nring, rb, d, bar);
                }
                if (jend > p) {   // the step's own token, read from the caller's buffers
                    const int o2 = off + (nring > 0 ? nring : 0);
                    umma::bulk_g2s(kd + (size_t)o2 * rb, kin, rb, bar);
                    umma::bulk_g2s(vd + (size_t)o2 * rb, vin, rb, bar);
                }
            }
        } else if (it < IT.nkc + IT.nlc) {
            const long long j0 = IT.jlo + (long long)(it - IT.nkc) * 16;
            const int nl = (int)min(16LL, IT.lhi - j0);
            const uint32_t fb = (uint32_t)(D * E);
            umma::mbar_arrive_expect_tx(bar, (uint32_t)nl * (fb + rb));
            ring_rows(buf, (const T *)phiV + (size_t)lam * D, j0, nl, fb, D, bar);
            ring_rows(buf + 16 * fb, VR, j0, nl, rb, d, bar);
        } else {
            const int r0 = (it - IT.nkc - IT.nlc) * 32;
            umma::mbar_arrive_expect_tx(bar, (uint32_t)(32 * d * 4 + 128));
            umma::bulk_g2s(buf, Hg + (size_t)r0 * d, (uint32_t)(32 * d * 4), bar);
            umma::bulk_g2s(buf + 32 * d * 4, sg + r0, 128u, bar);
        }
    };
    if (lane == 0)
        for (int k = 0; k < nst && k < nmine; ++k) issue(k, k);

    // ---- prologue: fates, raw rows, scaled queries; the appended pair joins the ring
    const bool phik = do_append && split == 0;
    const int nr = g + (phik ? 1 : 0);
    const T *qg = (const T *)a.q + ((size_t)b * dm.Hq + (size_t)hk * g) * d;
    const float scale = rsqrtf((float)d);
    const int nL = (int)(a.L_hi - a.L_lo);
    for (int i = tid; i < nL; i += nthr) fate[i] = S.pend[(size_t)st * dm.Lmax + i];
    for (int e = tid; e < nr * d; e += nthr) {
        const int r = e / d, c = e - r * d;
        const float x = to_f<T>(r < g ? qg[(size_t)r * d + c] : kin[c]);
        xs[r * d + c] = x;
        if (r < g) qs[r * QS + qidx<VN>(c)] = x * scale;
    }
    if (phik) {
        T *kr = (T *)S.KR + ((size_t)st * R + (p & (R - 1))) * d;
        T *vr = (T *)S.VR + ((size_t)st * R + (p & (R - 1))) * d;
        for (int c = tid; c < d; c += nthr) {
            kr[c] = kin[c];
            vr[c] = vin[c];
        }
    }
    __syncthreads();
    // z = x W for the nr rows: thread = (4 feature columns, a range of x dims); the
    // partial sums of a column group are reduced over the lanes that share it
    {
        const int ncg = Dh / 4;
        const int ncr = nthr / ncg >= 1 ? nthr / ncg : 1;   // power of two
        const int cg = tid / ncr, cr = tid % ncr;
        const int per = d / ncr;
        float z[kMaxG + 1][4];
#pragma unroll
        for (int r = 0; r <= kMaxG; ++r) z[r][0] = z[r][1] = z[r][2] = z[r][3] = 0.f;
        if (cg < ncg) {
#pragma unroll 8
            for (int c = cr * per; c < (cr + 1) * per; ++c) {
                const float4 w4 = __ldg((const float4 *)(S.W + (size_t)c * Dh) + cg);
#pragma unroll
                for (int r = 0; r <= kMaxG; ++r) {
                    if (r < nr) {
                        const float x = xs[r * d + c];
                        z[r][0] = fmaf(x, w4.x, z[r][0]);
                        z[r][1] = fmaf(x, w4.y, z[r][1]);
                        z[r][2] = fmaf(x, w4.z, z[r][2]);
                        z[r][3] = fmaf(x, w4.w, z[r][3]);
                    }
                }
            }
        }
        for (int o = 1; o < ncr; o <<= 1) {
#pragma unroll
            for (int r = 0; r <= kMaxG; ++r)
#pragma unroll
                for (int u = 0; u < 4; ++u) z[r][u] += __shfl_xor_sync(0xffffffffu, z[r][u], o);
        }
        if (cg < ncg && cr == 0) {
#pragma unroll
            for (int r = 0; r <= kMaxG; ++r)
                if (r < nr)
#pragma unroll
                    for (int u = 0; u < 4; ++u) zs[r * Dh + cg * 4 + u] = z[r][u];
        }
    }
    __syncthreads();
    for (int r = warp; r < nr; r += nw) {
        float zmax = -INFINITY, zmin = INFINITY;
        for (int i = lane; i < Dh; i += 32) {
            zmax = fmaxf(zmax, zs[r * Dh + i]);
            zmin = fminf(zmin, zs[r * Dh + i]);
        }
        zmax = warp_max(zmax);
        zmin = warp_min(zmin);
        float sp = 0.f, sn = 0.f;
        for (int i = lane; i < Dh; i += 32) {
            sp += __expf(zs[r * Dh + i] - zmax);
            sn += __expf(zmin - zs[r * Dh + i]);
        }
        const float rp = 1.f / warp_sum(sp), rn = 1.f / warp_sum(sn);
        for (int i = lane; i < Dh; i += 32) {
            const float fp = __expf(zs[r * Dh + i] - zmax) * rp;
            const float fn = __expf(zmin - zs[r * Dh + i]) * rn;
            if (r < g) {
                phq[r * PS + qidx<VN>(i)] = fp;
                phq[r * PS + qidx<VN>(Dh + i)] = fn;
            } else {
                T *pr = phiV + (size_t)(lam + (int)(p & (R - 1))) * D;
                pr[i] = from_f<T>(fp);
                pr[Dh + i] = from_f<T>(fn);
            }
        }
    }
    __syncthreads();

    // ---- per-warp accumulators: softmax (shift m >= 0) and the unscaled linear part
    float m[kMaxG], l[kMaxG], ld[kMaxG], o[kMaxG][DPL], lo[kMaxG][DPL];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        m[h] = 0.f;
        l[h] = 0.f;
        ld[h] = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) o[h][u] = lo[h][u] = 0.f;
    }
    bool ok = true;
    int kfail = nmine;
    for (int k = 0; k < nmine; ++k) {
        const int s = k % nst;
        const uint32_t par = (uint32_t)((k / nst) & 1);
        bool got = true;
        if (lane == 0) {
            const bool aborted = (*(volatile int *)S.err & ERR_TIMEOUT) != 0;
            got = !aborted && umma::mbar_wait(&mb[s], par, kWaitNs);
            if (!got) raise_error(S.err, ERR_TIMEOUT);
        }
        got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
        if (!got) {
            ok = false;
            kfail = k;
            break;
        }
        const int it = gw + k * wstride;
        const uint8_t *buf = ring + (size_t)s * SB;
        if (it < IT.nkc) {
            // ---- softmax keys
            const int k0 = it * 32, nk = min(32, IT.nsoft - k0);
            const int key = k0 + lane;
            bool soft = lane < nk;
            if (soft && key >= nS) {
                const long long j = IT.wlo + (key - nS);
                if (j >= a.L_lo && j < a.L_hi && fate[(int)(j - a.L_lo)] == 0) soft = false;   // kept: a cache slot
            }
            float sc[kMaxG];
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) sc[h] = 0.f;
            if (soft) {
                const uint8_t *kr = buf + (size_t)lane * d * E;
#pragma unroll 4
                for (int c = 0; c < CPR; ++c) {
                    const int c2 = c ^ (lane & XM);
                    float kf[VN];
                    Chunk<T>::load(kr + c2 * 16, kf);
#pragma unroll
                    for (int h = 0; h < kMaxG; ++h) {
                        if (h < g) {
                            const float *qh = qs + h * QS + qoff<VN>(c2, 0);
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
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h < g) {
                    const float s_ = soft ? sc[h] : -INFINITY;
                    const float mn = fmaxf(m[h], warp_max(s_));
                    const float f = __expf(m[h] - mn);
                    const float pw = soft ? __expf(s_ - mn) : 0.f;
                    l[h] = fmaf(l[h], f, warp_sum(pw));
#pragma unroll
                    for (int u = 0; u < DPL; ++u) o[h][u] *= f;
                    m[h] = mn;
                    pws[h * 32 + lane] = pw;
                }
            }
            __syncwarp();
            // P V: lane owns value dims [lane*DPL, lane*DPL + DPL)
            const uint8_t *vb = buf + (size_t)32 * d * E;
            for (int j0 = 0; j0 < nk; j0 += 4) {
                float4 w4[kMaxG];
#pragma unroll
                for (int h = 0; h < kMaxG; ++h)
                    if (h < g) w4[h] = *(const float4 *)(pws + h * 32 + j0);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if (j0 + t < nk) {
                        const T *vr = (const T *)(vb + (size_t)(j0 + t) * d * E);
                        float vf[DPL];
#pragma unroll
                        for (int u = 0; u < DPL; ++u) vf[u] = to_f<T>(vr[lane * DPL + u]);
#pragma unroll
                        for (int h = 0; h < kMaxG; ++h) {
                            if (h < g) {
                                const float wv = t == 0 ? w4[h].x : t == 1 ? w4[h].y : t == 2 ? w4[h].z : w4[h].w;
#pragma unroll
                                for (int u = 0; u < DPL; ++u) o[h][u] = fmaf(wv, vf[u], o[h][u]);
                            }
                        }
                    }
                }
            }
        } else if (it < IT.nkc + IT.nlc) {
            // ---- linear band: weights phi(q_h) . phi(k_j) of folded leaving pairs,
            //      lanes (key, half of the features), summed over the two halves
            const long long j0 = IT.jlo + (long long)(it - IT.nkc) * 16;
            const int nl = (int)min(16LL, IT.lhi - j0);
            const int kk = lane & 15, hf = lane >> 4;
            const bool lin = kk < nl && fate[(int)(j0 + kk - a.L_lo)] != 0;
            float gl[kMaxG];
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) gl[h] = 0.f;
            if (lin) {
                const uint8_t *fr = buf + (size_t)kk * D * E;
                const int cb = hf * (CPD >> 1);
                for (int c = 0; c < (CPD >> 1); ++c) {
                    const int c2 = cb + (c ^ (kk & XMD));
                    float ff[VN];
                    Chunk<T>::load(fr + c2 * 16, ff);
#pragma unroll
                    for (int h = 0; h < kMaxG; ++h) {
                        if (h < g) {
                            const float *ph = phq + h * PS + qoff<VN>(c2, 0);
#pragma unroll
                            for (int u = 0; u < VN; u += 4) {
                                const float4 q4 = *(const float4 *)(ph + u);
                                gl[h] = fmaf(q4.x, ff[u], gl[h]);
                                gl[h] = fmaf(q4.y, ff[u + 1], gl[h]);
                                gl[h] = fmaf(q4.z, ff[u + 2], gl[h]);
                                gl[h] = fmaf(q4.w, ff[u + 3], gl[h]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h < g) {
                    gl[h] += __shfl_xor_sync(0xffffffffu, gl[h], 16);
                    if (hf == 0) pws[h * 32 + kk] = gl[h];
                }
            }
            __syncwarp();
            const uint8_t *vb = buf + (size_t)16 * D * E;
            for (int jj = 0; jj < nl; ++jj) {
                const T *vr = (const T *)(vb + (size_t)jj * d * E);
                float vf[DPL];
#pragma unroll
                for (int u = 0; u < DPL; ++u) vf[u] = to_f<T>(vr[lane * DPL + u]);
#pragma unroll
                for (int h = 0; h < kMaxG; ++h) {
                    if (h < g) {
                        const float wv = pws[h * 32 + jj];
#pragma unroll
                        for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(wv, vf[u], lo[h][u]);
                        ld[h] += wv;
                    }
                }
            }
        } else {
            // ---- readout rows r0..r0+31: phi(q)^T H, phi(q)^T s (unscaled)
            const int r0 = (it - IT.nkc - IT.nlc) * 32;
            const float *Hs = (const float *)buf;
            const float *ss = (const float *)(buf + 32 * d * 4);
#pragma unroll 4
            for (int i = 0; i < 32; ++i) {
                float hv[DPL];
#pragma unroll
                for (int u = 0; u < DPL; ++u) hv[u] = Hs[i * d + lane * DPL + u];
                const float si = ss[i];
                const int fi = qidx<VN>(r0 + i);
#pragma unroll
                for (int h = 0; h < kMaxG; ++h) {
                    if (h < g) {
                        const float f = phq[h * PS + fi];
#pragma unroll
                        for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(f, hv[u], lo[h][u]);
                        ld[h] = fmaf(f, si, ld[h]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && k + nst < nmine) {
            fence_proxy_async();   // this buffer's reads are done before the copy overwrites it
            issue(k + nst, s);
        }
    }
    if (!ok && lane == 0) {
        // let the copies still in flight land before the buffers are reused (bounded)
        for (int k = kfail; k < kfail + nst && k < nmine; ++k)
            umma::mbar_wait(&mb[k % nst], (uint32_t)((k / nst) & 1), kWaitNs);
    }
    // every warp is past its staging buffers (the merge reuses them); a timed-out
    // wait anywhere in the CTA ends it here, with the error word set
    if (__syncthreads_or(ok ? 0 : 1)) return;

    // ---- merge the warps of this CTA
    const int rec_w = 3 + 2 * d;
    float *red = (float *)smd;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h < g) {
            float *rw = red + (size_t)(warp * kMaxG + h) * rec_w;
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
    for (int h = warp; h < g; h += nw) {
        float M = 0.f;
        for (int w = 0; w < nw; ++w) M = fmaxf(M, red[(w * kMaxG + h) * rec_w]);
        float Ls = 0.f, LD = 0.f, O[DPL], LO[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) O[u] = LO[u] = 0.f;
        for (int w = 0; w < nw; ++w) {
            const float *rw = red + (size_t)(w * kMaxG + h) * rec_w;
            const float f = __expf(rw[0] - M);
            Ls = fmaf(f, rw[1], Ls);
            LD += rw[2];
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                O[u] = fmaf(f, rw[3 + lane * DPL + u], O[u]);
                LO[u] += rw[3 + d + lane * DPL + u];
            }
        }
        if (dm.nsplit == 1) {
            const float em = __expf(-M);
            const float rden = 1.f / (Ls + em * (LD + dm.eps));
            T *out = (T *)a.out + ((size_t)b * dm.Hq + (size_t)hk * g + h) * d;
#pragma unroll
            for (int u = 0; u < DPL; ++u) out[lane * DPL + u] = from_f<T>((O[u] + em * LO[u]) * rden);
        } else {
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
    }
    if (dm.nsplit == 1) return;

    // ---- the last CTA of the stream merges the splits and writes the output
    __threadfence();
    __syncthreads();
    if (tid == 0) last_cta = atomicAdd(&S.dec_cnt[st], 1) == dm.nsplit - 1 ? 1 : 0;
    __syncthreads();
    if (!last_cta) return;
    __threadfence();
    for (int h = warp; h < g; h += nw) {
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
        T *out = (T *)a.out + ((size_t)b * dm.Hq + (size_t)hk * g + h) * d;
#pragma unroll
        for (int u = 0; u < DPL; ++u) out[lane * DPL + u] = from_f<T>((O[u] + em * LO[u]) * rden);
    }
    if (tid == 0) S.dec_cnt[st] = 0;
}

// Appends the step's key/value to the window ring (one CTA per stream) and,
// with with_phi, writes phi(k) of it into the phi rows (warp 0).
template <typename T>
__global__ void append_kernel(Dims dm, DevState S, const T *__restrict__ k, const T *__restrict__ v,
                              long long pos, int with_phi)
{
    __shared__ float xs[128];
    const int st = blockIdx.x;
    const int slot = (int)(pos & (dm.R - 1));
    T *KR = (T *)S.KR + ((size_t)st * dm.R + slot) * dm.d;
    T *VR = (T *)S.VR + ((size_t)st * dm.R + slot) * dm.d;
    for (int c = threadIdx.x; c < dm.d; c += blockDim.x) {
        KR[c] = k[(size_t)st * dm.d + c];
        VR[c] = v[(size_t)st * dm.d + c];
    }
    if (with_phi && threadIdx.x < 32)
        phi_row_warp<T>(k + (size_t)st * dm.d, S.W, xs, dm.d, dm.Dh,
                        (T *)S.phiV + ((size_t)st * (dm.lam + dm.R) + dm.lam + slot) * dm.D);
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

size_t decode_smem_bytes(const Dims &dm) { return dec_layout(dm).total; }

bool decode_plan(Dims *dm)
{
    const int e = dm->dtype == 0 ? 4 : 2;
    const size_t sb_keys = (size_t)32 * 2 * dm->d * e;
    const size_t sb_lin = (size_t)16 * (dm->D + dm->d) * e;
    const size_t sb_h = (size_t)32 * dm->d * 4 + 128;
    size_t sb = sb_keys > sb_h ? sb_keys : sb_h;
    if (sb_lin > sb) sb = sb_lin;
    dm->dec_sb = (int)((sb + 127) / 128 * 128);
    // shape with the most staging bytes in flight per SM (buffers beyond the one
    // being worked on), at up to 228 KB of shared memory per SM
    const int shapes[6][2] = {{2, 3}, {4, 3}, {4, 2}, {2, 2}, {1, 3}, {1, 2}};
    long long best = -1;
    int bw = 0, bs = 0, bres = 1;
    for (auto &sh : shapes) {
        dm->dec_nw = sh[0];
        dm->dec_nst = sh[1];
        const size_t tot = dec_layout(*dm).total;
        if (tot > 200 * 1024) continue;
        int res = (int)((228 * 1024) / (tot + 1024));
        if (res > 16 / sh[0]) res = 16 / sh[0];       // registers: ~170 per thread
        const long long fly = (long long)res * sh[0] * (sh[1] - 1) * dm->dec_sb;
        if (fly > best) {
            best = fly;
            bw = sh[0];
            bs = sh[1];
            bres = res;
        }
    }
    if (best < 0) return false;
    dm->dec_nw = bw;
    dm->dec_nst = bs;
    // about two waves of resident CTAs, at least one item per warp
    const long long nkeys = (long long)dm->lam + dm->eta + 1;
    const long long items = (nkeys + 31) / 32 + (dm->Cdec + 15) / 16 + dm->D / 32;
    const long long want = 2LL * kSMs * bres;
    long long nsp = (want + dm->ns - 1) / dm->ns;
    const long long cap = (items + bw - 1) / bw;
    if (nsp > cap) nsp = cap;
    if (nsp < 1) nsp = 1;
    dm->nsplit = (int)nsp;
    return true;
}

void launch_decode_append(const Dims &dm, const DevState &S, const void *k, const void *v,
                          long long pos, int with_phi, cudaStream_t stream)
{
    if (dm.dtype == 0)
        append_kernel<float><<<dm.ns, 128, 0, stream>>>(dm, S, (const float *)k, (const float *)v, pos,
                                                        with_phi);
    else
        append_kernel<__nv_bfloat16><<<dm.ns, 128, 0, stream>>>(
            dm, S, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, pos, with_phi);
}

void launch_decode_attn(const Dims &dm, const DevState &S, const DecodeArgs &a, int do_append,
                        cudaStream_t stream)
{
    dim3 grid(dm.nsplit, dm.ns);
    const size_t smem = dec_layout(dm).total;
    const int threads = 32 * dm.dec_nw;
#define LOLA_DECODE3(T, DPL)                                                                       \
    do {                                                                                           \
        static size_t attr = 0;   /* largest opt-in set so far */                                 \
        if (smem > attr) {                                                                         \
            cudaFuncSetAttribute(decode3_kernel<T, DPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 (int)smem);                                                       \
            attr = smem;                                                                           \
        }                                                                                          \
        decode3_kernel<T, DPL><<<grid, threads, smem, stream>>>(dm, S, a, do_append);              \
    } while (0)
    if (dm.dtype == 0) {
        if (dm.d == 32) LOLA_DECODE3(float, 1);
        else if (dm.d == 64) LOLA_DECODE3(float, 2);
        else LOLA_DECODE3(float, 4);
    } else {
        if (dm.d == 32) LOLA_DECODE3(__nv_bfloat16, 1);
        else if (dm.d == 64) LOLA_DECODE3(__nv_bfloat16, 2);
        else LOLA_DECODE3(__nv_bfloat16, 4);
    }
#undef LOLA_DECODE3
}

void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream)
{
    get_indices_kernel<<<64, 256, 0, stream>>>(dm, S, nS, idx, cnt);
}

}  // namespace lola
