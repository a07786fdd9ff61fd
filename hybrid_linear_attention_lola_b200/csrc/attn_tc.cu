// Tensor-core prefill output of a LoLA hybrid-attention layer for bfloat16
// inputs (gist.science technical summary, "Inferentiestrategie": linear
// attention + sparse-cache attention + sliding-window attention, combined).
//
// One CTA = one update interval of one (batch, kv-head) stream and 128 query
// rows; row r is (position t0 + mt*128/g + r/g, query head hk*g + r%g), so the
// rows of a tile are consecutive in q and out. Row r is TMEM lane r; threads
// r and r + 128 (the two halves of the CTA) share it, each exponentiating half
// of every 64-key tile.
//   1. O = phi(Q) [H'|s']   (readout of the interval's snapshot; column d of O
//      carries the linear denominator phi(q).s', so it rescales with O);
//   2. per 64-key tile: S = Q K^T (and G = phi(Q) phi(K)^T for window tiles that
//      hold folded leaving pairs) on the tensor cores; P = e^{s-m} for softmax
//      keys and g e^{-m} for linear keys, with the running shift
//      m = max(0, max score); O is rescaled in TMEM when m grows; O += P V.
//      Tile i+1's keys and values are copied while tile i is processed.
//   3. out = O[:, :d] / (sum P + O[:, d] + eps e^{-m}).
// Key classes: cached keys are softmax (causal); window keys [t0 - eta, t1)
// are softmax while inside the window of p, linear once they left it and were
// folded, and skipped when they were kept (they appear among the cached keys).
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {

namespace {

using bf16 = __nv_bfloat16;
constexpr int kThreads = 256;
constexpr int KT = 64;                // keys per tile
constexpr float kLazy = 8.f;          // shift slack of the lazy rescaling (natural log units)
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per tensor-core completion wait
enum : int { INFO_SOFT = 0, INFO_FOLDED = 1, INFO_SKIP = 2 };

struct TileMeta {
    int tok[KT], info[KT], vrow[KT];
    int lin[2];        // per producing warp: some key is a folded leaving pair
    int causal[2];     // per producing warp: every key is causal for every row of the CTA
    int nk, band;
};

struct AGeo {
    int d, D, FP, NB, NBa;
    uint32_t ncols;
    size_t off_phq, off_big, off_K[2], off_V[2], off_phk, off_P, off_wt, off_meta, off_red, total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline AGeo make_ageo(const Dims &dm)
{
    AGeo g{};
    g.d = dm.d;
    g.D = dm.D;
    g.FP = (dm.D + 127) / 128 * 128;
    g.NB = dm.d + 16;
    g.NBa = (g.NB + 31) / 32 * 32;
    const uint32_t need = (uint32_t)(g.NBa + 2 * KT);
    g.ncols = need <= 128 ? 128 : need <= 256 ? 256 : 512;
    const int dp = (g.d + 63) / 64 * 64;                  // K-major rows span whole atoms
    size_t o = (size_t)128 * dp * 2;                       // Q
    g.off_phq = al(o, 1024);
    o = g.off_phq + (size_t)128 * g.FP * 2;                // phi(Q)
    g.off_big = al(o, 1024);                               // snapshot image, then key tiles
    o = g.off_big;
    for (int b = 0; b < 2; ++b) {
        g.off_K[b] = al(o, 1024);
        g.off_V[b] = al(g.off_K[b] + (size_t)KT * dp * 2, 1024);
        o = g.off_V[b] + (size_t)KT * g.d * 2;
    }
    g.off_phk = al(o, 1024);
    g.off_P = al(g.off_phk + (size_t)KT * g.FP * 2, 1024);
    const size_t tiles_end = g.off_P + (size_t)128 * KT * 2;
    const size_t img_end = g.off_big + (size_t)g.FP * (g.d + 16) * 2;
    // W^T (K-major, Dh rows) behind the snapshot image: both are dead once the key tiles load
    g.off_wt = al(img_end, 1024);
    const size_t wt_end = g.off_wt + (size_t)(g.D / 2) * dp * 2;
    o = tiles_end > wt_end ? tiles_end : wt_end;
    g.off_meta = al(o, 16);
    g.off_red = al(g.off_meta + 2 * sizeof(TileMeta), 16);
    g.total = g.off_red + 128 * 4 + 1024;
    return g;
}

// Thread 0 waits for the MMA completion (bounded); a timeout anywhere in the
// grid sets the device error word, after which every CTA stops waiting.
__device__ __forceinline__ bool wait_mbar(uint64_t *mbar, uint32_t &phase, int *okflag, int *err)
{
    if (threadIdx.x == 0) {
        const bool aborted = (*(volatile int *)err & ERR_TIMEOUT) != 0;
        const bool ok = !aborted && umma::mbar_wait(mbar, phase, kWaitNs);
        if (!ok) raise_error(err, ERR_TIMEOUT);
        *okflag = ok ? 1 : 0;
    }
    __syncthreads();
    phase ^= 1u;
    umma::fence_after_sync();
    return *okflag != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(Dims dm, DevState S, PrefillScratch P, AttnArgs a, KVSrc<bf16> src)
{
    const AGeo g = make_ageo(dm);
    const int d = g.d, D = g.D, FP = g.FP, eta = dm.eta, lam = dm.lam, gq = dm.g;
    const int tiles_per_int = (dm.C * gq + 127) / 128;
    const int ci = a.ci0 + blockIdx.x / tiles_per_int, mt = blockIdx.x % tiles_per_int;
    const int st = blockIdx.y;
    const int b = st / dm.Hkv, hk = st % dm.Hkv;
    const long long t0 = a.pos0 + (long long)ci * dm.C, t1 = t0 + dm.C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, half = warp >> 2;
    const int r = qd * 32 + lane;                    // this thread's row (TMEM lane)
    const int rows_total = dm.C * gq;
    const int grow = mt * 128 + r;
    const bool row_ok = grow < rows_total;
    const long long p = t0 + grow / gq;              // query position of the row
    const long long pmin = t0 + (mt * 128) / gq;     // smallest position in the CTA
    const float scale = rsqrtf((float)d);
    const int lgd = __ffs(d >> 3) - 1, lgf = __ffs(FP >> 3) - 1;   // 16-byte chunks per row

    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    __shared__ int okflag;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *sQ = base, *sPhq = base + g.off_phq, *sImg = base + g.off_big;
    uint8_t *sPhk = base + g.off_phk, *sP = base + g.off_P;
    TileMeta *meta = (TileMeta *)(base + g.off_meta);
    float *red = (float *)(base + g.off_red);

    if (tid == 0) umma::mbar_init(&mbar, 1);
    if (warp == 0) umma::tmem_alloc(&tslot, g.ncols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tm = tslot;
    const uint32_t tO = tm, tS = tm + (uint32_t)g.NBa, tG = tS + KT;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    uint32_t phase = 0;

    // ---- stage Q, W^T and the snapshot image
    const bf16 *q = (const bf16 *)a.q;
    const int Dh = D / 2;
    uint8_t *sWt = base + g.off_wt;
    const size_t qrow0 = ((size_t)b * a.n_call + (size_t)(t0 - a.pos0)) * dm.Hq + (size_t)hk * gq;
    for (int e = tid; e < (128 << lgd); e += kThreads) {
        const int rr = e >> lgd, kc = e & ((1 << lgd) - 1);
        const int gr = mt * 128 + rr;
        uint8_t *dst = sQ + umma::kmajor_offset(rr, kc * 8, 128);
        if (gr < rows_total) {
            const size_t row = qrow0 + (size_t)(gr / gq) * dm.Hq + gr % gq;
            umma::cp_async16(dst, q + row * d + kc * 8);
        } else {
            *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
    }
    {
        const bf16 *Wt = (const bf16 *)S.Wt;
        for (int e = tid; e < (Dh << lgd); e += kThreads) {
            const int rr = e >> lgd, kc = e & ((1 << lgd) - 1);
            umma::cp_async16(sWt + umma::kmajor_offset(rr, kc * 8, Dh), Wt + (size_t)rr * d + kc * 8);
        }
    }
    {
        const int nb = FP * (d + 16) * 2;
        const uint8_t *img = (const uint8_t *)P.snapImg + ((size_t)st * dm.mmax + ci) * nb;
        for (int e = tid; e < nb / 16; e += kThreads) umma::cp_async16(sImg + e * 16, img + e * 16);
    }
    umma::cp_async_commit();
    umma::cp_async_wait_all();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();

    bool ok = true;
    // ---- 0. phi(Q) = [softmax(Q W), softmax(-Q W)]: Z = Q W on the tensor cores (into the
    //         score columns), then each row's two softmaxes; half 0 of the CTA writes the
    //         first Dh features, half 1 the last Dh, as bf16 into the K-major phi(Q) tile
    if (tid == 0) {
        umma::fence_after_sync();
        const uint32_t q0 = umma::smem_u32(sQ), w0 = umma::smem_u32(sWt);
        const uint32_t id_z = umma::idesc_bf16(128, Dh, false, false);
        for (int ks = 0; ks < d / 16; ++ks)
            umma::mma_ss(tS, umma::kmajor_desc(q0, ks, 128), umma::kmajor_desc(w0, ks, Dh), id_z,
                         ks > 0 ? 1u : 0u);
        umma::mma_commit(&mbar);
    }
    ok = wait_mbar(&mbar, phase, &okflag, S.err);
    if (ok) {
        float zmax = -INFINITY, zmin = INFINITY;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                zmax = fmaxf(zmax, v[j]);
                zmin = fminf(zmin, v[j]);
            }
        }
        float ssum = 0.f;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) ssum += half ? __expf(zmin - v[j]) : __expf(v[j] - zmax);
        }
        const float rs_ = 1.f / ssum;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; j += 8) {
                float f[8];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    f[t] = (half ? __expf(zmin - v[j + t]) : __expf(v[j + t] - zmax)) * rs_;
                uint4 pk;
                pk.x = umma::pack_bf16x2(f[0], f[1]);
                pk.y = umma::pack_bf16x2(f[2], f[3]);
                pk.z = umma::pack_bf16x2(f[4], f[5]);
                pk.w = umma::pack_bf16x2(f[6], f[7]);
                *(uint4 *)(sPhq + umma::kmajor_offset(r, half * Dh + c0 + j, 128)) = pk;
            }
        }
        if (half == 1)
            for (int c = D; c < FP; c += 8)
                *(uint4 *)(sPhq + umma::kmajor_offset(r, c, 128)) = make_uint4(0, 0, 0, 0);
    }
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();

    // ---- 1. O = phi(Q) [H'|s']: the snapshot holds H' as an N-contiguous [FP][d]
    //         operand followed by s' as row 0 of a K-major 16 x FP operand
    if (tid == 0 && ok) {
        umma::fence_after_sync();
        const uint32_t a0 = umma::smem_u32(sPhq), bh = umma::smem_u32(sImg);
        const uint32_t bs = bh + (uint32_t)(FP * d * 2);
        const uint32_t id_h = umma::idesc_bf16(128, d, false, true);
        const uint32_t id_s = umma::idesc_bf16(128, 16, false, false);
        for (int ks = 0; ks < FP / 16; ++ks) {
            const uint64_t ad = umma::kmajor_desc(a0, ks, 128);
            umma::mma_ss(tO, ad, umma::mnmajor_desc(bh, ks, d), id_h, ks > 0 ? 1u : 0u);
            umma::mma_ss(tO + (uint32_t)d, ad, umma::kmajor_desc(bs, ks, 16), id_s, ks > 0 ? 1u : 0u);
        }
        umma::mma_commit(&mbar);
    }
    if (ok) ok = wait_mbar(&mbar, phase, &okflag, S.err);

    const size_t lb = (size_t)st * dm.mmax + ci;
    const int nK = P.logCount[lb];
    const int *ltok = P.logTok + lb * lam;
    const int *lvrow = P.logVrow + lb * lam;
    const uint8_t *llf = P.logLf + lb * dm.Lmax;
    const long long jlo = t0 - eta > 0 ? t0 - eta : 0;
    const int nband = (int)(t1 - jlo);
    const int ntb = (nband + KT - 1) / KT, ntc = (nK + KT - 1) / KT;
    const int ntiles = ntb + ntc;
    const uint32_t id_s = umma::idesc_bf16(128, KT, false, false);
    const uint32_t id_pv = umma::idesc_bf16(128, d, false, true);
    const bf16 *phiK = (const bf16 *)P.phiK + (size_t)st * (lam + dm.R + dm.Nmax) * D;

    // metadata of tile i (threads 0..63, i.e. warps 0 and 1)
    auto fill_meta = [&](int i, TileMeta &M) {
        const bool band = i < ntb;
        const long long kb = band ? jlo + (long long)i * KT : (long long)(i - ntb) * KT;
        const int nk = band ? (int)min((long long)KT, t1 - kb) : min(KT, nK - (int)kb);
        int tok = -1, info = INFO_SKIP, vr = 0;
        if (tid < nk) {
            if (band) {
                const long long j = kb + tid;
                tok = (int)j;
                vr = src.tok2vrow(j);
                info = (j < t1 - eta) ? (llf[(int)(j - (t0 - eta))] ? INFO_FOLDED : INFO_SKIP) : INFO_SOFT;
            } else {
                tok = ltok[kb + tid];
                vr = lvrow[kb + tid];
                info = INFO_SOFT;
            }
        }
        M.tok[tid] = tok;
        M.info[tid] = info;
        M.vrow[tid] = vr;
        const bool l_any = __any_sync(0xffffffffu, info == INFO_FOLDED);
        const bool c_all = __all_sync(0xffffffffu, tid < nk && tok <= pmin);
        if (lane == 0) {
            M.lin[warp] = l_any ? 1 : 0;
            M.causal[warp] = (!band && c_all) ? 1 : 0;
        }
        if (tid == 0) {
            M.nk = nk;
            M.band = band ? 1 : 0;
        }
    };
    // copies of tile i's keys, values and (for linear keys) phi(K) into buffer bf
    auto issue_copies = [&](const TileMeta &M, int bf) {
        uint8_t *sK = base + g.off_K[bf], *sV = base + g.off_V[bf];
        const int nk = M.nk;
        for (int e = tid; e < (KT << lgd); e += kThreads) {
            const int j = e >> lgd, kc = e & ((1 << lgd) - 1);
            uint8_t *dk = sK + umma::kmajor_offset(j, kc * 8, KT);
            uint8_t *dv = sV + umma::mnmajor_offset(j, kc * 8, d);
            if (j < nk) {
                const int vr = M.vrow[j];
                umma::cp_async16(dk, src.krow(st, vr) + kc * 8);
                umma::cp_async16(dv, src.vrow(st, vr) + kc * 8);
            } else {
                *(uint4 *)dk = make_uint4(0, 0, 0, 0);
                *(uint4 *)dv = make_uint4(0, 0, 0, 0);
            }
        }
        if (M.lin[0] | M.lin[1]) {
            for (int e = tid; e < (KT << lgf); e += kThreads) {
                const int j = e >> lgf, kc = e & ((1 << lgf) - 1);
                uint8_t *dst = sPhk + umma::kmajor_offset(j, kc * 8, KT);
                if (j < nk && kc * 8 < D) umma::cp_async16(dst, phiK + (size_t)M.vrow[j] * D + kc * 8);
                else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
            }
        }
        umma::cp_async_commit();
    };

    float m = 0.f, lpart = 0.f;
    // QK^T (and, for tiles with folded band keys, phi(Q) phi(K)^T) of tile t into TMEM
    auto issue_scores = [&](int t) {
        const TileMeta &M = meta[t & 1];
        const uint32_t q0 = umma::smem_u32(sQ), k0 = umma::smem_u32(base + g.off_K[t & 1]);
        for (int ks = 0; ks < d / 16; ++ks)
            umma::mma_ss(tS, umma::kmajor_desc(q0, ks, 128), umma::kmajor_desc(k0, ks, KT), id_s, ks > 0 ? 1u : 0u);
        if (M.lin[0] | M.lin[1]) {
            const uint32_t pq0 = umma::smem_u32(sPhq), pk0 = umma::smem_u32(sPhk);
            for (int ks = 0; ks < FP / 16; ++ks)
                umma::mma_ss(tG, umma::kmajor_desc(pq0, ks, 128), umma::kmajor_desc(pk0, ks, KT), id_s,
                             ks > 0 ? 1u : 0u);
        }
    };
    if (ntiles > 0 && ok) {
        if (tid < KT) fill_meta(0, meta[0]);
        __syncthreads();
        issue_copies(meta[0], 0);
        if (ntiles > 1 && tid < KT) fill_meta(1, meta[1]);
        umma::cp_async_wait_all();
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            issue_scores(0);
            umma::mma_commit(&mbar);
        }
    }
    const int nch = g.NB / 16, split = (nch + 1) / 2;   // O chunks rescaled by half 0 / half 1
    // Per tile i, one completion wait: it covers QK^T(i) and PV(i-1), which were
    // committed together. Then tile i+1's rows load while tile i's softmax runs, and
    // PV(i) and QK^T(i+1) go to the tensor cores together.
    for (int i = 0; i < ntiles && ok; ++i) {
        const TileMeta &M = meta[i & 1];
        if (!(ok = wait_mbar(&mbar, phase, &okflag, S.err))) break;
        // buffers (i+1)&1 held tile i-1, whose MMAs are complete
        if (i + 1 < ntiles) issue_copies(meta[(i + 1) & 1], (i + 1) & 1);
        const bool lin = (M.lin[0] | M.lin[1]) != 0;

        // ---- softmax / linear weights; this half exponentiates keys [32*half, 32*half + 32)
        float sv[KT];
#pragma unroll
        for (int c0 = 0; c0 < KT; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) sv[c0 + j] = v[j] * scale;
        }
        const bool fast = (M.causal[0] & M.causal[1]) != 0;
        float tmax = -INFINITY;
        if (fast) {
#pragma unroll
            for (int j = 0; j < KT; ++j) tmax = fmaxf(tmax, sv[j]);
        } else {
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                const int info = M.info[j], tok = M.tok[j];
                const bool soft = info != INFO_SKIP && tok <= p && !(info == INFO_FOLDED && tok <= p - eta);
                if (soft) tmax = fmaxf(tmax, sv[j]);
            }
        }
        // lazy rescaling: the shift m only moves when the row's maximum exceeds it by
        // more than kLazy (weights stay below e^kLazy; numerator and denominator share m)
        const bool grow_m = tmax > m + kLazy;
        if (__any_sync(0xffffffffu, grow_m)) {
            // TMEM accesses are warp-collective: the whole warp rescales its chunk range
            const float f = grow_m ? __expf(m - tmax) : 1.f;
            lpart *= f;
            const int cb = half ? split : 0, ce = half ? nch : split;
            for (int cc = cb; cc < ce; ++cc) {
                float v[16];
                umma::tmem_ld16(tO + lane_off + (uint32_t)(cc * 16), v);
                umma::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] *= f;
                umma::tmem_st16(tO + lane_off + (uint32_t)(cc * 16), v);
            }
            umma::tmem_wait_st();
            if (grow_m) m = tmax;
        }
        float gv[32];
        if (lin) {
#pragma unroll
            for (int c0 = 0; c0 < 32; c0 += 16) {
                float v[16];
                umma::tmem_ld16(tG + lane_off + (uint32_t)(half * 32 + c0), v);
                umma::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) gv[c0 + j] = v[j];
            }
        }
        const float em = __expf(-m);
        float rs = 0.f;
#pragma unroll
        for (int j0 = 0; j0 < 32; j0 += 8) {
            float pf[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int k = j0 + jj, j = half * 32 + k;
                const float s = half ? sv[32 + k] : sv[k];   // static indices keep sv in registers
                float pw;
                if (fast) {
                    pw = __expf(s - m);
                } else {
                    const int info = M.info[j], tok = M.tok[j];
                    pw = 0.f;
                    if (info != INFO_SKIP && tok <= p) {
                        if (info == INFO_FOLDED && tok <= p - eta) pw = lin ? gv[k] * em : 0.f;
                        else pw = __expf(s - m);
                    }
                }
                pf[jj] = row_ok ? pw : 0.f;
            }
            uint4 pk;
            pk.x = umma::pack_bf16x2(pf[0], pf[1]);
            pk.y = umma::pack_bf16x2(pf[2], pf[3]);
            pk.z = umma::pack_bf16x2(pf[4], pf[5]);
            pk.w = umma::pack_bf16x2(pf[6], pf[7]);
            // the row sum uses the rounded weights the tensor core multiplies
            rs += umma::bf16lo_to_f32(pk.x) + umma::bf16hi_to_f32(pk.x) + umma::bf16lo_to_f32(pk.y) +
                  umma::bf16hi_to_f32(pk.y) + umma::bf16lo_to_f32(pk.z) + umma::bf16hi_to_f32(pk.z) +
                  umma::bf16lo_to_f32(pk.w) + umma::bf16hi_to_f32(pk.w);
            *(uint4 *)(sP + umma::kmajor_offset(r, half * 32 + j0, 128)) = pk;
        }
        lpart += rs;
        // tile i+1's rows (issued above) have landed; P is written
        umma::cp_async_wait_all();
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t p0 = umma::smem_u32(sP), v0 = umma::smem_u32(base + g.off_V[i & 1]);
            for (int ks = 0; ks < KT / 16; ++ks)
                umma::mma_ss(tO, umma::kmajor_desc(p0, ks, 128), umma::mnmajor_desc(v0, ks, d), id_pv, 1u);
            if (i + 1 < ntiles) issue_scores(i + 1);
            umma::mma_commit(&mbar);
        }
        // meta[i & 1] is free (every thread is past tile i's softmax): tile i+2's metadata
        if (i + 2 < ntiles && tid < KT) fill_meta(i + 2, meta[i & 1]);
    }
    // the last PV
    if (ok && ntiles > 0) ok = wait_mbar(&mbar, phase, &okflag, S.err);
    umma::cp_async_wait_all();

    if (ok) {
        // ---- 3. normalise and store; half h writes value columns [h*d/2, (h+1)*d/2)
        if (half == 1) red[r] = lpart;
        __syncthreads();
        const float l = half == 0 ? lpart + red[r] : 0.f;
        __syncthreads();
        if (half == 0) red[r] = l;
        __syncthreads();
        const float lt = red[r];
        float v[16];
        umma::tmem_ld16(tO + lane_off + (uint32_t)d, v);
        umma::tmem_wait_ld();
        const float den = lt + v[0] + dm.eps * __expf(-m);
        const float rden = 1.f / den;
        bf16 *out = (bf16 *)a.out;
        const size_t orow = qrow0 + (size_t)(grow / gq) * dm.Hq + grow % gq;
        for (int c0 = half * (d / 2); c0 < (half + 1) * (d / 2); c0 += 16) {
            umma::tmem_ld16(tO + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
            if (row_ok) {
                uint4 o0, o1;
                o0.x = umma::pack_bf16x2(v[0] * rden, v[1] * rden);
                o0.y = umma::pack_bf16x2(v[2] * rden, v[3] * rden);
                o0.z = umma::pack_bf16x2(v[4] * rden, v[5] * rden);
                o0.w = umma::pack_bf16x2(v[6] * rden, v[7] * rden);
                o1.x = umma::pack_bf16x2(v[8] * rden, v[9] * rden);
                o1.y = umma::pack_bf16x2(v[10] * rden, v[11] * rden);
                o1.z = umma::pack_bf16x2(v[12] * rden, v[13] * rden);
                o1.w = umma::pack_bf16x2(v[14] * rden, v[15] * rden);
                *(uint4 *)(out + orow * d + c0) = o0;
                *(uint4 *)(out + orow * d + c0 + 8) = o1;
            }
        }
    } else if (tid == 0) {
        raise_error(S.err, ERR_TIMEOUT);
        umma::mbar_wait(&mbar, phase ^ 1u, kWaitNs);
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tm, g.ncols);
}

}  // namespace

size_t attn_tc_smem_bytes(const Dims &dm) { return make_ageo(dm).total; }

void launch_attn_tc(const Dims &dm, const DevState &S, const PrefillScratch &P, const AttnArgs &a,
                    cudaStream_t stream)
{
    KVSrc<bf16> src{(const bf16 *)S.KS, (const bf16 *)S.VS, (const bf16 *)S.KR, (const bf16 *)S.VR,
                    (const bf16 *)a.kin, (const bf16 *)a.vin, dm.lam, dm.R, a.n_call, dm.Hkv, dm.d,
                    a.pos0};
    const int tiles_per_int = (dm.C * dm.g + 127) / 128;
    dim3 grid(a.m * tiles_per_int, dm.ns);
    const size_t smem = make_ageo(dm).total;
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_tc_kernel<<<grid, kThreads, smem, stream>>>(dm, S, P, a, src);
}

}  // namespace lola
