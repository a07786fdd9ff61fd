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
// A step streams everything it reads once from HBM. bfloat16: a preparation
// kernel computes phi(q) and appends the new pair; the streaming kernel, launched
// as its programmatic dependent, cuts every stream's work into items -- key chunks
// (32 keys: their key and value rows, 128-byte-swizzled TMA tiles), linear-band
// chunks (16 leaving pairs: phi and value rows) and state chunks (16 feature rows
// of H and s) -- and gives every warp a contiguous run of the items of all
// streams, staged through the warp's own ring of shared-memory buffers (one
// mbarrier per buffer) while it works on the current one. A key chunk is one
// mma.sync m16n8k16 pass for Q K^T (the group's heads as the M rows) and one for
// P V, the score fragments reused as the P operand; band and state chunks run on
// the CUDA cores. A warp leaving a stream writes its partial (shift, softmax and
// linear sums per head); the warp that writes a stream's last partial merges them
// (a per-stream counter). float32: one kernel (decode3_kernel) does the same with
// SIMT scores and a per-CTA split of each stream.
#include "lola_internal.cuh"
#include "umma.cuh"

#include <cudaTypedefs.h>

namespace lola {

namespace {

constexpr int kMaxG = 8;
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s per staging-buffer wait
constexpr int kSMs = 148;
constexpr int kMinPer = 8;   // items per warp of the streaming kernel, at least (many streams)
#ifndef LOLA_DEC_MINPER_FLOOR
#define LOLA_DEC_MINPER_FLOOR 1
#endif
constexpr int kMinPerFloor = LOLA_DEC_MINPER_FLOOR;   // ... and with few streams
#ifndef LOLA_DECODE_BUFS
#define LOLA_DECODE_BUFS 2
#endif
constexpr int kStreamBufs = LOLA_DECODE_BUFS;   // staging buffers per warp of the streaming kernel
constexpr int kFewBufs = 4;   // ... when the streams are too few to fill the GPU with warps
constexpr int kFewPer = 6;    // items per warp, at least, in that case

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
//   [nkc, nkc + nlc)    16 linear-band tokens of [jlo, lhi), pairs leaving the window
//                       this interval (kept ones are skipped): with state_ahead the
//                       folded ones still inside p's window (the state holds their
//                       linear terms, which come off; the softmax attends them),
//                       otherwise the folded ones that left it (their terms add)
//   [nkc + nlc, ni)     hrows feature rows of the state (H, s)
// With tma, softmax keys come in aligned 32-row blocks instead: cache slots
// [32c, 32c + 32) (c < ncc), then the blocks of 32 ring slots the window
// [wlo, p] touches (nwc of them, from block wblk0 on, modulo R / 32); rows of a
// block outside the key set are masked.
struct Items {
    long long jlo, wlo, lhi;
    int nsoft, nkc, nlc, ni;
    int ncc, nwc, wblk0;
};

__host__ __device__ __forceinline__ Items make_items(const Dims &dm, const DecodeArgs &a, int hrows, int tma)
{
    Items it;
    const long long p = a.pos;
    const long long jl = a.t0 - dm.eta > 0 ? a.t0 - dm.eta : 0;   // first pair leaving in the interval
    it.wlo = p - dm.eta + 1 > jl ? p - dm.eta + 1 : jl;
    if (a.state_ahead) {
        // folded pairs still inside the window: their linear terms come off the state
        it.jlo = it.wlo;
        it.lhi = a.L_hi > it.jlo ? a.L_hi : it.jlo;
    } else {
        // folded pairs that left the window: their linear terms add to the state
        it.jlo = jl;
        it.lhi = a.L_hi < it.wlo ? a.L_hi : it.wlo;
        if (it.lhi < it.jlo) it.lhi = it.jlo;
    }
    const int nwin = (int)(p - it.wlo + 1);
    it.nsoft = a.nS + nwin;
    it.ncc = (a.nS + 31) / 32;
    it.nwc = 0;
    it.wblk0 = 0;
    if (tma) {
        if (nwin > 0) {
            const int f = (int)(it.wlo & (dm.R - 1)) >> 5, l = (int)(p & (dm.R - 1)) >> 5;
            it.nwc = ((l - f) & ((dm.R >> 5) - 1)) + 1;
            it.wblk0 = f;
        }
        it.nkc = it.ncc + it.nwc;
    } else {
        it.nkc = (it.nsoft + 31) / 32;
    }
    it.nlc = (int)((it.lhi - it.jlo + 15) / 16);
    it.ni = it.nkc + it.nlc + dm.D / hrows;
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
    const Items IT = make_items(dm, a, 32, 0);
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
                const float4 w4 = __ldg((const float4 *)(w_of(dm, S.W, st % dm.Hkv) + (size_t)c * Dh) + cg);
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
            got = umma::mbar_wait_abortable(&mb[s], par, kWaitNs, S.err, ERR_TIMEOUT);
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
                    if (hf == 0) pws[h * 32 + kk] = a.state_ahead ? -gl[h] : gl[h];
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


// ---------------------------------------------------------------- bfloat16: warp-level MMA
//
// Same items and pipeline as above, staged with 16-byte cp.async into a
// 128-byte XOR-swizzled row layout (conflict-free ldmatrix). For a chunk of 32
// keys, S = Q K^T and O += P V run as mma.sync m16n8k16 (bf16 in, fp32
// accumulate) with the group's heads as the M rows (padded to 16); the score
// fragments become the P operand directly. Linear-band and state items use the
// SIMT code of the kernel above.

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// C[16x8] += A[16x16] B[16x8]; rows 8..15 of A are zero (a1 = a3 = 0)
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// byte offset of 16-byte chunk c of row r in a [32 rows][CPR chunks] swizzled tile
// DPL consecutive floats (16-, 8- or 4-byte aligned) through L2
template <int DPL> __device__ __forceinline__ void ld_dpl(const float *p, float (&v)[DPL])
{
    if constexpr (DPL == 4) {
        const float4 x = __ldcg((const float4 *)p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else if constexpr (DPL == 2) {
        const float2 x = __ldcg((const float2 *)p);
        v[0] = x.x; v[1] = x.y;
    } else {
#pragma unroll
        for (int u = 0; u < DPL; ++u) v[u] = __ldcg(p + u);
    }
}

template <int CPR> __device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)((c >> 3) * 32 * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Launches `kernel` as a programmatic dependent of the previous kernel on the stream:
// it may start while that one still runs and orders itself with griddep_wait().
template <typename... P, typename... A>
void launch_dependent(void (*kernel)(P...), int grid, int block, size_t smem, cudaStream_t stream, A... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Step preparation (bfloat16 path): phi(q) of every query row into an fp32
// scratch, and, when the step appends, the new pair into the window ring with
// phi(k) of it in the phi rows. One warp per row; W (fp32) in shared memory.
// The streaming kernel that follows is launched as a programmatic dependent: it
// starts at once and waits for this grid only before it reads phi(q) or the
// appended pair.
template <typename T>
__global__ void __launch_bounds__(256) decode_prep_kernel(Dims dm, DevState S, DecodeArgs a, int do_append)
{
    umma::griddep_launch_dependents();
    extern __shared__ float smp[];
    const int d = dm.d, Dh = dm.Dh, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *Ws = smp;
    float *xs = smp + d * Dh + warp * d;
    const int hw = blockIdx.y;   // with one W per kv-head, grid row hw takes that kv-head's rows
    const bool by_head = gridDim.y > 1;
    {
        // 16-byte copies, all in flight at once (d * Dh is a multiple of 4)
        const float4 *w4 = (const float4 *)(S.W + (size_t)hw * d * Dh);
        float4 *s4 = (float4 *)Ws;
        const int n4 = d * Dh / 4;
#pragma unroll 4
        for (int e = threadIdx.x; e < n4; e += blockDim.x) s4[e] = __ldg(w4 + e);
    }
    __syncthreads();
    const int nq = by_head ? dm.B * dm.g : dm.B * dm.Hq, nk = do_append ? (by_head ? dm.B : dm.ns) : 0;
    const int slot = (int)(a.pos & (dm.R - 1));
    for (int rr = blockIdx.x * 8 + warp; rr < nq + nk; rr += gridDim.x * 8) {
        if (rr < nq) {
            const int r = by_head ? (rr / dm.g) * dm.Hq + hw * dm.g + rr % dm.g : rr;
            phi_row_warp<T, float>((const T *)a.q + (size_t)r * d, Ws, xs, d, Dh, S.phiQd + (size_t)r * dm.D);
        } else {
            const int st = by_head ? (rr - nq) * dm.Hkv + hw : rr - nq;
            const T *k = (const T *)a.k + (size_t)st * d, *v = (const T *)a.v + (size_t)st * d;
            T *kr = (T *)S.KR + ((size_t)st * dm.R + slot) * d, *vr = (T *)S.VR + ((size_t)st * dm.R + slot) * d;
            for (int c = lane; c < d; c += 32) {
                kr[c] = k[c];
                vr[c] = v[c];
            }
            phi_row_warp<T, T>(k, Ws, xs, d, Dh, (T *)S.phiV + ((size_t)st * (dm.lam + dm.R) + dm.lam + slot) * dm.D);
        }
    }
}

// Streaming decode (bfloat16 path). A persistent grid; the work items of all
// streams form one list (stream-major, see make_items) and every warp takes a
// contiguous range of it, flowing its items through its own ring of
// shared-memory buffers (two by default): 32-key chunks of cache and window as
// tiled TMA loads with 128-byte swizzle (d = 64 or 128; other d as bulk copies of
// padded rows), linear-band rows and state rows as bulk copies, each completing on
// the buffer's mbarrier. For a chunk of 32 keys,
// S = Q K^T and O += P V run as mma.sync m16n8k16 (bf16 in, fp32 accumulate)
// with the group's heads as the M rows (padded to 16); the score fragments become
// the P operand directly. Linear band and state items run on the SIMT units. When
// a warp leaves a stream it writes its partial (m, l, linear den, softmax num,
// linear num per head); the warp that writes a stream's last partial merges them
// (a per-stream counter).
template <int DPL, int G, int NST>
__global__ void __launch_bounds__(128) decode_stream_kernel(Dims dm, DevState S, DecodeArgs a, int per, int wbytes,
                                                             const __grid_constant__ DecMaps maps)
{
    using T = __nv_bfloat16;
    constexpr int d = 32 * DPL;
    constexpr int E = 2;
    constexpr int VN = 8;
    constexpr int CPR = d / 8;                         // 16-byte chunks per key row
    constexpr int KS_ = d / 16;                        // k-steps of Q K^T
    constexpr int ND = d / 8;                          // n-tiles of P V (8 value dims each)
    constexpr int HR = 16;                             // state rows per item
    constexpr int RS = d * E + 16;                     // padded row stride of key / value tiles (bulk path)
    const bool tma = dm.dec_tma != 0;
    // bytes of a 32-row key (or value) tile: swizzled 128-byte rows (TMA path) or padded rows
    const int KTB = tma ? 32 * 128 * ((CPR + 7) / 8) : 32 * RS;
    const int SB = dm.dec_sb;
    const int nw = blockDim.x >> 5;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, tig = lane & 3;          // fragment row (head) and column pair
    const int D = dm.D, g = dm.g, lam = dm.lam, R = dm.R;
    const long long p = a.pos;
    const int nS = a.nS;
    const Items IT = make_items(dm, a, HR, dm.dec_tma);
    const int ni = IT.ni;
    const long long total = (long long)dm.ns * ni;
    const long long gw = (long long)blockIdx.x * nw + warp;
    const long long i0 = gw * per;
    if (i0 >= total) return;                            // warp-uniform; no CTA-wide barriers below
    const int nmine = (int)min((long long)per, total - i0);
    const int PS = D;                                   // phi(q) row stride (floats; plain rows)
    const int CPD = D / VN;
    const int XMD = CPD >= 16 ? 7 : (CPD >> 1) - 1;
    const float scale = rsqrtf((float)d);

    extern __shared__ __align__(128) uint8_t smraw_d[];
    // 1024-byte aligned base: the 128-byte swizzle of TMA boxes is address based
    uint8_t *smd = smraw_d + (((umma::smem_u32(smraw_d) + 1023u) & ~1023u) - umma::smem_u32(smraw_d));
    uint8_t *wbase = smd + (size_t)warp * wbytes;
    uint8_t *ring = wbase;
    float *phq = (float *)(wbase + NST * SB);            // [G][D], filled by a bulk copy per stream
    float *pws = phq + G * PS;                           // [G][32]
    uint8_t *fate = (uint8_t *)(pws + G * 32);           // [Lmax]
    uint64_t *mb = (uint64_t *)(fate + 256);             // [NST] staging buffers, [NST] phi(q)

    // ---- copies of item k of this warp into buffer s: bulk (TMA) copies, completion
    //      counted on the buffer's mbarrier. Key chunks: one copy per key row and per
    //      value row into padded rows (stride RS: conflict-free ldmatrix), invalid rows
    //      zeroed. Linear-band and state items: contiguous row runs, plain layout.
    auto issue = [&](int k, int s) {
        if (k >= nmine) return;
        const long long gi = i0 + k;
        const int st = (int)(gi / ni), it = (int)(gi % ni);
        uint8_t *buf = ring + (size_t)s * SB;
        uint64_t *bar = &mb[s];
        if (it < IT.nkc && tma) {
            if (lane == 0) {
                const bool cache = it < IT.ncc;
                if (!cache) umma::griddep_wait();   // window rows include the pair the preparation appends
                const int y = cache ? it * 32 : ((IT.wblk0 + (it - IT.ncc)) & ((R >> 5) - 1)) * 32;
                const CUtensorMap *mk = cache ? &maps.ks : &maps.kr;
                const CUtensorMap *mv = cache ? &maps.vs : &maps.vr;
                const int nbox = (d + 63) / 64;
                umma::mbar_arrive_expect_tx(bar, (uint32_t)(nbox * 2 * 4096));
                for (int bx = 0; bx < nbox; ++bx) {
                    umma::tma_load_3d(buf + bx * 4096, mk, bx * 64, y, st, bar);
                    umma::tma_load_3d(buf + KTB + bx * 4096, mv, bx * 64, y, st, bar);
                }
            }
        } else if (it < IT.nkc) {
            const int k0 = it * 32;
            const int nv = min(32, IT.nsoft - k0);
            if (k0 + 32 > nS) umma::griddep_wait();   // window rows (the appended pair among them)
            if (lane == 0) umma::mbar_arrive_expect_tx(bar, (uint32_t)nv * 2 * d * E);
            __syncwarp();
            uint8_t *kd = buf + (size_t)lane * RS, *vd = buf + KTB + (size_t)lane * RS;
            const int key = k0 + lane;
            if (lane < nv) {
                const T *kr, *vr;
                if (key < nS) {
                    kr = (const T *)S.KS + ((size_t)st * lam + key) * d;
                    vr = (const T *)S.VS + ((size_t)st * lam + key) * d;
                } else {
                    const long long j = IT.wlo + (key - nS);
                    kr = (const T *)S.KR + ((size_t)st * R + (j & (R - 1))) * d;
                    vr = (const T *)S.VR + ((size_t)st * R + (j & (R - 1))) * d;
                }
                umma::bulk_g2s(kd, kr, (uint32_t)(d * E), bar);
                umma::bulk_g2s(vd, vr, (uint32_t)(d * E), bar);
            } else {
#pragma unroll
                for (int c = 0; c < CPR; ++c) {
                    *(uint4 *)(kd + c * 16) = make_uint4(0, 0, 0, 0);
                    *(uint4 *)(vd + c * 16) = make_uint4(0, 0, 0, 0);
                }
            }
        } else if (lane == 0) {
            if (it < IT.nkc + IT.nlc) {
                const long long j0 = IT.jlo + (long long)(it - IT.nkc) * 16;
                const int nl = (int)min(16LL, IT.lhi - j0);
                const uint32_t fb = (uint32_t)(D * E), rb = (uint32_t)(d * E);
                umma::mbar_arrive_expect_tx(bar, (uint32_t)nl * (fb + rb));
                const T *phiR = (const T *)S.phiV + ((size_t)st * (lam + R) + lam) * D;
                const T *VR = (const T *)S.VR + (size_t)st * R * d;
                uint8_t *fd = buf, *vd = buf + 16 * fb;
                long long j = j0;
                int n = nl;
                while (n > 0) {
                    const int slot = (int)(j & (R - 1));
                    const int m = min(n, R - slot);
                    umma::bulk_g2s(fd, phiR + (size_t)slot * D, (uint32_t)m * fb, bar);
                    umma::bulk_g2s(vd, VR + (size_t)slot * d, (uint32_t)m * rb, bar);
                    fd += (size_t)m * fb;
                    vd += (size_t)m * rb;
                    j += m;
                    n -= m;
                }
            } else {
                const int r0 = (it - IT.nkc - IT.nlc) * HR;
                umma::mbar_arrive_expect_tx(bar, (uint32_t)(HR * d * 4 + HR * 4));
                umma::bulk_g2s(buf, S.H + ((size_t)st * D + r0) * d, (uint32_t)(HR * d * 4), bar);
                umma::bulk_g2s(buf + HR * d * 4, S.s + (size_t)st * D + r0, (uint32_t)(HR * 4), bar);
            }
        }
    };
    if (lane == 0)
        for (int i = 0; i <= NST + 1; ++i) umma::mbar_init(&mb[i], 1);   // mb[NST + 1]: nothing arrives
    __syncwarp();
    for (int k = 0; k < NST; ++k) issue(k, k);

    // ---- per-stream state of this warp
    int cur = -1;
    uint32_t nbeg = 0;      // streams begun (phase of the phi(q) barrier)
    bool need_q = false;    // phi(q) of the current stream not yet waited for
    uint32_t qa0[KS_], qa2[KS_];
    float mrow = 0.f, lrow = 0.f;
    float oc[ND][4];
    float ld[G], lo[G][DPL];
    // false: the wait for the previous stream's phi(q) copy gave up (error word set)
    auto begin = [&](int st) -> bool {
        const int b = st / dm.Hkv, hk = st % dm.Hkv;
        // linear-band or state items of st in this warp's range need phi(q); a warp with
        // only key chunks of st neither copies it nor waits for the preparation
        const long long st_end = min((long long)st * ni + ni, i0 + nmine);
        const bool wantq = (int)(st_end - 1 - (long long)st * ni) >= IT.nkc;
        const T *qg = (const T *)a.q + ((size_t)b * dm.Hq + (size_t)hk * g) * d;
        const bool hv = gq < g;
#pragma unroll
        for (int ks = 0; ks < KS_; ++ks) {
            qa0[ks] = hv ? *(const uint32_t *)(qg + (size_t)gq * d + ks * 16 + tig * 2) : 0u;
            qa2[ks] = hv ? *(const uint32_t *)(qg + (size_t)gq * d + ks * 16 + 8 + tig * 2) : 0u;
        }
        // phi(q) of the group's heads: one bulk copy, waited for before the first
        // linear-band or state item of the stream (key chunks come first)
        fence_proxy_async();   // earlier reads of phq are done before the copy overwrites it
        __syncwarp();
        bool okq = true;
        if (lane == 0) {
            // a copy whose stream needed no phi(q) lands before the next one is issued
            if (need_q) {
                okq = umma::mbar_wait(&mb[NST], (nbeg - 1) & 1u, kWaitNs);
                if (!okq) raise_error(S.err, ERR_TIMEOUT);
            }
            if (okq && wantq) {
                umma::griddep_wait();   // phi(q) is written by the preparation grid
                umma::mbar_arrive_expect_tx(&mb[NST], (uint32_t)(g * D * 4));
                umma::bulk_g2s(phq, S.phiQd + ((size_t)b * dm.Hq + (size_t)hk * g) * D, (uint32_t)(g * D * 4),
                               &mb[NST]);
            }
        }
        if (__shfl_sync(0xffffffffu, okq ? 1 : 0, 0) == 0) return false;
        need_q = false;   // the previous stream's copy has landed (waited for above)
        if (wantq) {
            ++nbeg;
            need_q = true;
        }
        const int nL = (int)(a.L_hi - a.L_lo);
        for (int i = lane; i < nL; i += 32) fate[i] = S.pend[(size_t)st * dm.Lmax + i];
        mrow = 0.f;
        lrow = 0.f;
#pragma unroll
        for (int n = 0; n < ND; ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            ld[h] = 0.f;
#pragma unroll
            for (int u = 0; u < DPL; ++u) lo[h][u] = 0.f;
        }
        __syncwarp();
        return true;
    };
    // Leaves the step after a wait gave up (the error word is set): lets the copies
    // in flight land, item k's included (an abort does not wait for it).
    auto drain = [&](int k) {
        if (lane == 0) {
            for (int k2 = k; k2 < k + NST && k2 < nmine; ++k2)
                umma::mbar_wait(&mb[k2 % NST], (uint32_t)((k2 / NST) & 1), kWaitNs);
            if (need_q) umma::mbar_wait(&mb[NST], (nbeg - 1) & 1u, kWaitNs);
        }
        __syncwarp();
    };
    const size_t rec = 2 * d + 4;
    auto flush = [&](int st) {
        const long long first = ((long long)st * ni) / per;            // first warp with items of st
        const long long last = ((long long)st * ni + ni - 1) / per;
        const int nparts = (int)(last - first + 1), pi = (int)(gw - first);
        float lq = lrow + __shfl_xor_sync(0xffffffffu, lrow, 1);
        lq += __shfl_xor_sync(0xffffffffu, lq, 2);
        float *base = S.part + (size_t)st * dm.nsplit * g * rec;
        if (gq < g) {
            float *pr = base + ((size_t)pi * g + gq) * rec;
            if (tig == 0) {
                pr[0] = mrow;
                pr[1] = lq;
                pr[3] = 0.f;
            }
#pragma unroll
            for (int n = 0; n < ND; ++n) {
                pr[4 + n * 8 + tig * 2] = oc[n][0];
                pr[4 + n * 8 + tig * 2 + 1] = oc[n][1];
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if (h < g) {
                float *pr = base + ((size_t)pi * g + h) * rec;
                if (lane == 0) pr[2] = ld[h];
#pragma unroll
                for (int u = 0; u < DPL; ++u) pr[4 + d + lane * DPL + u] = lo[h][u];
            }
        }
        // publish the partial (release) and count it; the last one acquires all the others
        __syncwarp();
        int prev = 0;
        if (lane == 0)
            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(&S.dec_cnt[st]) : "memory");
        prev = __shfl_sync(0xffffffffu, prev, 0);
        __syncwarp();
        if (prev != nparts - 1) return;
        // this warp wrote the stream's last partial: merge (online-softmax identity) and write out
        const int b = st / dm.Hkv, hk = st % dm.Hkv;
        float Mh[G], Lsh[G], LDh[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            Mh[h] = 0.f;
            Lsh[h] = LDh[h] = 0.f;
            if (h >= g) continue;
            // lane q holds partials q, q + 32, ...: maximum shift and the scalar sums in parallel
            for (int q2 = lane; q2 < nparts; q2 += 32) Mh[h] = fmaxf(Mh[h], __ldcg(base + ((size_t)q2 * g + h) * rec));
            Mh[h] = warp_max(Mh[h]);
            for (int q2 = lane; q2 < nparts; q2 += 32) {
                const float *pr = base + ((size_t)q2 * g + h) * rec;
                Lsh[h] = fmaf(__expf(__ldcg(pr) - Mh[h]), __ldcg(pr + 1), Lsh[h]);
                LDh[h] += __ldcg(pr + 2);
            }
            Lsh[h] = warp_sum(Lsh[h]);
            LDh[h] = warp_sum(LDh[h]);
        }
        // value columns: lane owns dims [lane*DPL, lane*DPL + DPL); one head at a time, four
        // partials in flight, DPL floats per load
        for (int h = 0; h < g; ++h) {
            float O[DPL], LO[DPL];
#pragma unroll
            for (int u = 0; u < DPL; ++u) O[u] = LO[u] = 0.f;
            float M = 0.f, Ls = 0.f, LD = 0.f;
#pragma unroll
            for (int h2 = 0; h2 < G; ++h2)
                if (h2 == h) {
                    M = Mh[h2];
                    Ls = Lsh[h2];
                    LD = LDh[h2];
                }
            for (int q0 = 0; q0 < nparts; q0 += 4) {
                float mv[4], ov[4][DPL], lv[4][DPL];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int q2 = q0 + t < nparts ? q0 + t : q0;
                    const float *pr = base + ((size_t)q2 * g + h) * rec;
                    mv[t] = __ldcg(pr);
                    ld_dpl<DPL>(pr + 4 + lane * DPL, ov[t]);
                    ld_dpl<DPL>(pr + 4 + d + lane * DPL, lv[t]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if (q0 + t < nparts) {
                        const float f = __expf(mv[t] - M);
#pragma unroll
                        for (int u = 0; u < DPL; ++u) {
                            O[u] = fmaf(f, ov[t][u], O[u]);
                            LO[u] += lv[t][u];
                        }
                    }
                }
            }
            const float em = __expf(-M);
            const float rden = 1.f / (Ls + em * (LD + dm.eps));
            T *out = (T *)a.out + ((size_t)b * dm.Hq + (size_t)hk * g + h) * d;
#pragma unroll
            for (int u = 0; u < DPL; ++u) out[lane * DPL + u] = from_f<T>((O[u] + em * LO[u]) * rden);
        }
        if (lane == 0) S.dec_cnt[st] = 0;
    };

    if (a.inject_ns != 0 && gw == 0) {
        // test hook: a bounded wait that runs out, handled like any other timeout (the
        // warp leaves before counting its partial)
        bool got = true;
        if (lane == 0) {
            got = umma::mbar_wait(&mb[NST + 1], 0, a.inject_ns);
            if (!got) raise_error(S.err, ERR_TIMEOUT);
        }
        if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
            drain(0);
            return;
        }
    }
    for (int k = 0; k < nmine; ++k) {
        const int s = k % NST;
        const long long gi = i0 + k;
        const int st = (int)(gi / ni), it = (int)(gi % ni);
        if (st != cur) {
            if (cur >= 0) flush(cur);
            if (!begin(st)) {
                drain(k);
                return;
            }
            cur = st;
        }
        bool got = true;
        if (lane == 0) {
            got = umma::mbar_wait_abortable(&mb[s], (uint32_t)((k / NST) & 1), kWaitNs, S.err, ERR_TIMEOUT);
            if (!got) raise_error(S.err, ERR_TIMEOUT);
        }
        if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
            drain(k);
            return;
        }
        const uint8_t *buf = ring + (size_t)s * SB;
        if (it >= IT.nkc && need_q) {
            bool okq = true;
            if (lane == 0) {
                okq = umma::mbar_wait(&mb[NST], (nbeg - 1) & 1u, kWaitNs);
                if (!okq) raise_error(S.err, ERR_TIMEOUT);
            }
            if (__shfl_sync(0xffffffffu, okq ? 1 : 0, 0) == 0) {
                need_q = false;   // that copy was waited for (and given up on) just now
                drain(k);
                return;
            }
            need_q = false;
        }
        if (it < IT.nkc) {
            bool soft;
            long long j = -1;   // window token of this lane's row, if any
            if (tma) {
                if (it < IT.ncc) {
                    soft = it * 32 + lane < nS;
                } else {
                    const int slot = ((IT.wblk0 + (it - IT.ncc)) & ((R >> 5) - 1)) * 32 + lane;
                    j = IT.wlo + ((slot - (int)(IT.wlo & (R - 1))) & (R - 1));
                    soft = j <= p;
                }
            } else {
                const int key = it * 32 + lane;
                soft = key < IT.nsoft;
                if (soft && key >= nS) j = IT.wlo + (key - nS);
            }
            if (soft && j >= 0 && j >= a.L_lo && j < a.L_hi && fate[(int)(j - a.L_lo)] == 0)
                soft = false;   // kept leaving pair: attended as a cache slot
            const unsigned smask = __ballot_sync(0xffffffffu, soft);
            const uint32_t kb = umma::smem_u32(buf), vb = kb + KTB;
            float sc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
            const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
#pragma unroll
                for (int kp = 0; kp < KS_; ++kp) {
                    const int krow = np * 16 + (mi >> 1) * 8 + rr;
                    const int kch = kp * 2 + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb + (tma ? swz<CPR>(krow, kch) : (uint32_t)(krow * RS + kch * 16)), b0, b1, b2, b3);
                    mma16816(sc[np * 2], qa0[kp], qa2[kp], b0, b1);
                    mma16816(sc[np * 2 + 1], qa0[kp], qa2[kp], b2, b3);
                }
            }
            float cmax = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    sc[nt][e] *= scale;
                    if ((smask >> (nt * 8 + tig * 2 + e)) & 1u) cmax = fmaxf(cmax, sc[nt][e]);
                }
            cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
            cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
            const float mn = fmaxf(mrow, cmax);
            const float f = __expf(mrow - mn);
            mrow = mn;
            lrow *= f;
#pragma unroll
            for (int n = 0; n < ND; ++n) {
                oc[n][0] *= f;
                oc[n][1] *= f;
            }
            uint32_t pa[4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float p0 = ((smask >> (nt * 8 + tig * 2)) & 1u) ? __expf(sc[nt][0] - mn) : 0.f;
                const float p1 = ((smask >> (nt * 8 + tig * 2 + 1)) & 1u) ? __expf(sc[nt][1] - mn) : 0.f;
                pa[nt] = pack2(p0, p1);
                lrow += umma::bf16lo_to_f32(pa[nt]) + umma::bf16hi_to_f32(pa[nt]);
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int n = 0; n < ND; n += 2) {
                    const int vrow = kk * 16 + (mi & 1) * 8 + rr;
                    const int vch = n + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vb + (tma ? swz<CPR>(vrow, vch) : (uint32_t)(vrow * RS + vch * 16)), b0, b1, b2, b3);
                    mma16816(oc[n], pa[kk * 2], pa[kk * 2 + 1], b0, b1);
                    mma16816(oc[n + 1], pa[kk * 2], pa[kk * 2 + 1], b2, b3);
                }
            }
        } else if (it < IT.nkc + IT.nlc) {
            const long long j0 = IT.jlo + (long long)(it - IT.nkc) * 16;
            const int nl = (int)min(16LL, IT.lhi - j0);
            const int kk = lane & 15, hf = lane >> 4;
            const bool lin = kk < nl && fate[(int)(j0 + kk - a.L_lo)] != 0;
            float gl[G];
#pragma unroll
            for (int h = 0; h < G; ++h) gl[h] = 0.f;
            if (lin) {
                const uint8_t *fr = buf + (size_t)kk * D * E;
                const int cb = hf * (CPD >> 1);
                for (int c = 0; c < (CPD >> 1); ++c) {
                    const int c2 = cb + (c ^ (kk & XMD));
                    float ff[VN];
                    Chunk<T>::load(fr + c2 * 16, ff);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        if (h < g) {
                            const float *ph = phq + h * PS + c2 * VN;
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
            for (int h = 0; h < G; ++h) {
                if (h < g) {
                    gl[h] += __shfl_xor_sync(0xffffffffu, gl[h], 16);
                    if (hf == 0) pws[h * 32 + kk] = lin ? (a.state_ahead ? -gl[h] : gl[h]) : 0.f;
                }
            }
            __syncwarp();
            const uint8_t *vbp = buf + (size_t)16 * D * E;
            for (int jj = 0; jj < nl; ++jj) {
                const T *vr = (const T *)(vbp + (size_t)jj * d * E);
                float vf[DPL];
#pragma unroll
                for (int u = 0; u < DPL; ++u) vf[u] = to_f<T>(vr[lane * DPL + u]);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (h < g) {
                        const float wv = pws[h * 32 + jj];
#pragma unroll
                        for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(wv, vf[u], lo[h][u]);
                        ld[h] += wv;
                    }
                }
            }
        } else {
            const int r0 = (it - IT.nkc - IT.nlc) * HR;
            const float *Hs = (const float *)buf;
            const float *ss = (const float *)(buf + HR * d * 4);
#pragma unroll 4
            for (int i = 0; i < HR; ++i) {
                float hv[DPL];
#pragma unroll
                for (int u = 0; u < DPL; ++u) hv[u] = Hs[i * d + lane * DPL + u];
                const float si = ss[i];
                const int fi = r0 + i;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (h < g) {
                        const float fq = phq[h * PS + fi];
#pragma unroll
                        for (int u = 0; u < DPL; ++u) lo[h][u] = fmaf(fq, hv[u], lo[h][u]);
                        ld[h] = fmaf(fq, si, ld[h]);
                    }
                }
            }
        }
        __syncwarp();
        fence_proxy_async();   // this buffer's reads are done before the copies overwrite it
        issue(k + NST, s);
    }
    flush(cur);
    if (need_q && lane == 0) umma::mbar_wait(&mb[NST], (nbeg - 1) & 1u, kWaitNs);   // no copy outlives the warp
}

// bytes of shared memory per warp of decode_stream_kernel
inline int stream_warp_bytes(const Dims &dm, int G)
{
    const size_t b = (size_t)dm.dec_nst * dm.dec_sb + (size_t)G * (dm.D + dm.D / 8) * 4 + (size_t)G * 32 * 4 + 256 + 64;
    return (int)((b + 1023) / 1024 * 1024);   // every warp's buffers start 1024-byte aligned
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
        phi_row_warp<T, T>(k + (size_t)st * dm.d, w_of(dm, S.W, st % dm.Hkv), xs, dm.d, dm.Dh,
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
    if (dm->dtype != 0) {
        // streaming kernel: 3 buffers per warp of key chunks (2 swizzled 32-row tiles),
        // linear-band items (16 phi rows + 16 value rows) or state items (16 H rows + s)
        dm->dec_tma = (dm->d == 64 || dm->d == 128) && dm->R >= 32 ? 1 : 0;
        const size_t sb_keys = dm->dec_tma ? (size_t)2 * 32 * 128 * (dm->d / 64)
                                           : (size_t)2 * 32 * (dm->d * 2 + 16);
        const size_t sb_lin = (size_t)16 * (dm->D + dm->d) * 2;
        const size_t sb_h = (size_t)16 * dm->d * 4 + 64;
        size_t sb = sb_keys > sb_h ? sb_keys : sb_h;
        if (sb_lin > sb) sb = sb_lin;
        dm->dec_sb = (int)((sb + 1023) / 1024 * 1024);
        // aligned 32-row blocks: the cache and up to two more blocks for the window
        const long long items = ((long long)dm->lam + 31) / 32 + (dm->eta + 31) / 32 + 2 +
                                (dm->Cdec + 15) / 16 + dm->D / 16;
        // items per warp that would spread the streams over every SM; with fewer streams
        // than that, each warp keeps more copies in flight and takes at least kFewPer items
        // (the partials of a stream are merged by one warp: fewer, larger partials)
        long long mp = (long long)dm->ns * items / ((long long)kSMs * 8);
        const bool few = mp < kMinPer;
        dm->dec_nst = few ? kFewBufs : kStreamBufs;
        if (few && mp < kFewPer) mp = kFewPer;
        if (mp < kMinPerFloor) mp = kMinPerFloor;
        if (mp > kMinPer) mp = kMinPer;
        const int G = dm->g <= 1 ? 1 : dm->g <= 2 ? 2 : dm->g <= 4 ? 4 : 8;
        // warps per CTA: the most resident warps per SM (shared memory, ~160 registers per thread)
        const size_t wb = (size_t)stream_warp_bytes(*dm, G);
        int best = 0;
        dm->dec_nw = 0;
        for (int nw = 4; nw >= 1; --nw) {
            if ((size_t)nw * wb + 1024 > 227 * 1024) continue;
            int res = (int)((228 * 1024) / (nw * wb + 1024 + 1280));
            const int rlim = 65536 / (nw * 32 * 160);
            if (res > rlim) res = rlim;
            if (res * nw > best) {
                best = res * nw;
                dm->dec_nw = nw;
            }
        }
        if (dm->dec_nw == 0) return false;
        dm->dec_minper = (int)mp;
        dm->nsplit = (int)((items + mp - 1) / mp + 1);
        return true;
    }
    dm->dec_tma = 0;
    const int e = 4;
    const int hrows = 32;
    const size_t sb_keys = (size_t)32 * 2 * dm->d * e;
    const size_t sb_lin = (size_t)16 * (dm->D + dm->d) * e;
    const size_t sb_h = (size_t)hrows * dm->d * 4 + (size_t)hrows * 4;
    size_t sb = sb_keys > sb_h ? sb_keys : sb_h;
    if (sb_lin > sb) sb = sb_lin;
    dm->dec_sb = (int)((sb + 127) / 128 * 128);
    // shape with the most staging bytes in flight per SM (buffers beyond the one
    // being worked on), at up to 228 KB of shared memory per SM
    const int shapes[6][2] = {{4, 3}, {2, 3}, {4, 2}, {2, 2}, {1, 3}, {1, 2}};
    long long best = -1;
    int bw = 0, bs = 0, bres = 1;
    for (auto &sh : shapes) {
        dm->dec_nw = sh[0];
        dm->dec_nst = sh[1];
        const size_t tot = dec_layout(*dm).total;
        if (tot > 200 * 1024) continue;
        int res = (int)((228 * 1024) / (tot + 1024 + 256));   // + driver and static shared memory
        if (res > 16 / sh[0]) res = 16 / sh[0];                 // registers
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
    const long long items = (nkeys + 31) / 32 + (dm->Cdec + 15) / 16 + dm->D / hrows;
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
                        const DecMaps *maps, cudaStream_t stream)
{
    if (dm.dtype != 0) {
        // bfloat16: preparation, then the persistent streaming kernel
        const size_t psm = sizeof(float) * ((size_t)dm.d * dm.Dh + 8 * dm.d);
        {
            static size_t attr = 0;
            if (psm > attr) {
                cudaFuncSetAttribute(decode_prep_kernel<__nv_bfloat16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
                attr = psm;
            }
            const int rows = (dm.B * dm.Hq + (do_append ? dm.ns : 0)) / dm.nW;
            int grid = (rows + 7) / 8;
            if (grid > kSMs * 4) grid = kSMs * 4;
            decode_prep_kernel<__nv_bfloat16><<<dim3(grid, dm.nW), 256, psm, stream>>>(dm, S, a, do_append);
        }
        const int G = dm.g <= 1 ? 1 : dm.g <= 2 ? 2 : dm.g <= 4 ? 4 : 8;
        const int wb = stream_warp_bytes(dm, G);
        const int nw = dm.dec_nw;
        const size_t smem = (size_t)nw * wb + 1024;   // + alignment slack
        DecMaps mp{};
        if (maps != nullptr) mp = *maps;
        int res = (int)((228 * 1024) / (smem + 1280));   // smem includes the alignment slack
        if (res < 1) res = 1;
        if (res > 65536 / (nw * 32 * 160)) res = 65536 / (nw * 32 * 160);
        const long long total = (long long)dm.ns * make_items(dm, a, 16, dm.dec_tma).ni;
        const long long warps_cap = (long long)kSMs * res * nw;
        long long per = (total + warps_cap - 1) / warps_cap;
        if (per < dm.dec_minper) per = dm.dec_minper;
        const long long nwarps = (total + per - 1) / per;
        const int grid = (int)((nwarps + nw - 1) / nw);
#define LOLA_STREAM_N(DPL, GG, NB)                                                                 \
    do {                                                                                           \
        static size_t attr = 0;                                                                    \
        if (smem > attr) {                                                                         \
            cudaFuncSetAttribute(decode_stream_kernel<DPL, GG, NB>,                                \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);          \
            attr = smem;                                                                           \
        }                                                                                          \
        launch_dependent(decode_stream_kernel<DPL, GG, NB>, grid, nw * 32, smem, stream, dm, S, a, (int)per, wb, mp); \
    } while (0)
#define LOLA_STREAM(DPL, GG)                                                                       \
    do {                                                                                           \
        if (dm.dec_nst == kFewBufs) LOLA_STREAM_N(DPL, GG, kFewBufs);                              \
        else LOLA_STREAM_N(DPL, GG, kStreamBufs);                                                  \
    } while (0)
#define LOLA_STREAM_G(DPL)                                                                         \
    do {                                                                                           \
        if (G == 1) LOLA_STREAM(DPL, 1);                                                           \
        else if (G == 2) LOLA_STREAM(DPL, 2);                                                      \
        else if (G == 4) LOLA_STREAM(DPL, 4);                                                      \
        else LOLA_STREAM(DPL, 8);                                                                  \
    } while (0)
        if (dm.d == 32) LOLA_STREAM_G(1);
        else if (dm.d == 64) LOLA_STREAM_G(2);
        else LOLA_STREAM_G(4);
#undef LOLA_STREAM_G
#undef LOLA_STREAM
#undef LOLA_STREAM_N
        return;
    }
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
    if (dm.d == 32) LOLA_DECODE3(float, 1);
    else if (dm.d == 64) LOLA_DECODE3(float, 2);
    else LOLA_DECODE3(float, 4);
#undef LOLA_DECODE3
}

bool make_decode_maps(const Dims &dm, const DevState &S, DecMaps *maps)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return false;
        encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    auto one = [&](CUtensorMap *m, void *base, int rows) {
        const cuuint64_t dims[3] = {(cuuint64_t)dm.d, (cuuint64_t)(rows > 0 ? rows : 1), (cuuint64_t)dm.ns};
        const cuuint64_t strides[2] = {(cuuint64_t)dm.d * 2, (cuuint64_t)dm.d * 2 * (rows > 0 ? rows : 1)};
        const cuuint32_t box[3] = {64, 32, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    return one(&maps->ks, S.KS, dm.lam) && one(&maps->vs, S.VS, dm.lam) && one(&maps->kr, S.KR, dm.R) &&
           one(&maps->vr, S.VR, dm.R);
}

void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream)
{
    get_indices_kernel<<<64, 256, 0, stream>>>(dm, S, nS, idx, cnt);
}

}  // namespace lola
