// Tensor-core prefill output of a LoLA hybrid-attention layer for bfloat16
// inputs (gist.science technical summary, "Inferentiestrategie": linear
// attention + sparse-cache attention + sliding-window attention, combined).
//
// One CTA = one update interval of one (batch, kv-head) stream and 128 query
// rows; row r is (position t0 + mt*128/g + r/g, query head hk*g + r%g), so the
// rows of a tile are consecutive in q and out. Row r is TMEM lane r; threads
// r and r + 128 (the two halves of the CTA) share it.
//
// Setup, all at shift m = 0:
//   phi(Q) = [softmax(QW), softmax(-QW)]  (Z = QW on the tensor cores);
//   O = phi(Q) H1                         (readout of the interval's snapshot: the
//                                          state at the interval's end, with every
//                                          pair the interval folds);
//   l = phi(Q).s1                         (linear denominator, CUDA cores);
//   O -= G V_L, l -= sum G                (folded leaving pairs still inside the
//                                          window of the query, which the softmax
//                                          attends: G = phi(Q) phi(K_L)^T, masked
//                                          per row).
// Main loop, per 64-key tile of softmax keys (window keys, then cached keys):
//   S = Q K^T on the tensor cores into one of two TMEM score buffers;
//   P = e^{s - m} with the running shift m = max(0, max score), O rescaled in
//   TMEM when m grows; O += P V. Scores of tile i+2 are computed while tile i's
//   softmax runs, and the key and value rows of later tiles load into a ring of
//   shared-memory buffers several tiles ahead.
// Finally out = O / (l + eps e^{-m}).
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
constexpr int kMaxBufs = 12;          // key + value tile buffers of the ring, at most
constexpr int kMaxPro = 8;            // tiles whose metadata the prologue loads (NK + 1), at most
enum : int { INFO_SOFT = 0, INFO_FOLDED = 1, INFO_SKIP = 2 };

struct TileMeta {
    int tok[KT], vrow[KT];
    unsigned char info[KT];
    unsigned skip32[2], fold32[2];   // per 32 keys: never a softmax key here / a folded leaving pair
    int maxtok32[2];                 // per 32 keys: largest token of a key that is not skipped
};

// bits 0..x set (none for x < 0, all for x >= 63)
__device__ __forceinline__ unsigned long long prefix_mask(long long x)
{
    return x < 0 ? 0ull : x >= 63 ? ~0ull : (2ull << x) - 1ull;
}

// Shared memory: [Q][ones][P region][ring region][tile metadata][row sums]
//   P region: two 128 x 64 weight tiles (P0, P1); during setup W^T, then phi(K_L)
//   ring region: nbuf tiles of 64 x d (K-major keys or N-contiguous values);
//   buffer 0 holds V_L during setup, buffers 1.. hold H' and phi(Q)
struct AGeo {
    int d, D, FP, Dh, NK, NV, nbuf, MS, NBa;
    uint32_t ncols;
    size_t tileb, off_ones, off_P, off_R, off_H, off_phq, off_meta, off_red, total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline AGeo make_ageo_n(const Dims &dm, int nbuf)
{
    AGeo g{};
    g.d = dm.d;
    g.D = dm.D;
    g.FP = (dm.D + 127) / 128 * 128;
    g.Dh = dm.D / 2;
    g.NBa = (g.d + 16 + 31) / 32 * 32;   // O (d columns) and the weight sums (column d)
    uint32_t need = (uint32_t)(g.NBa + 2 * KT);
    if ((uint32_t)(g.NBa + g.Dh) > need) need = (uint32_t)(g.NBa + g.Dh);
    g.ncols = need <= 128 ? 128 : need <= 256 ? 256 : 512;
    g.tileb = (size_t)KT * g.d * 2;
    g.nbuf = nbuf;
    g.NV = nbuf / 2;
    g.NK = nbuf - g.NV;
    g.MS = g.NK + 2;
    size_t o = (size_t)128 * g.d * 2;                        // Q (K-major, d = whole atoms)
    g.off_ones = al(o, 1024);                                 // K-major 16 x 64, row 0 ones
    o = g.off_ones + 16 * KT * 2;
    g.off_P = al(o, 1024);
    size_t pr = (size_t)2 * 128 * KT * 2;
    const size_t wt = (size_t)g.Dh * g.d * 2, phk = (size_t)KT * g.FP * 2;
    if (wt > pr) pr = wt;
    if (phk > pr) pr = phk;
    g.off_R = al(g.off_P + pr, 1024);
    g.off_H = g.off_R + g.tileb;                              // buffer 1
    g.off_phq = g.off_H + al((size_t)g.FP * g.d * 2, g.tileb);
    o = g.off_R + (size_t)nbuf * g.tileb;
    const size_t setup_end = g.off_phq + (size_t)128 * g.FP * 2;
    if (setup_end > o) o = setup_end;
    g.off_meta = al(o, 16);
    size_t ms = (size_t)g.MS * sizeof(TileMeta);
    if ((size_t)g.FP * 4 > ms) ms = (size_t)g.FP * 4;         // s' (fp32) during setup
    g.off_red = al(g.off_meta + ms, 16);
    g.total = g.off_red + 128 * 4 + 1024;                     // + alignment slack of the base
    if (g.NK + 1 > kMaxPro) g.total = (size_t)1 << 30;        // unsupported ring: never chosen
    return g;
}

// Buffers needed by the setup (V_L, H', phi(Q)), then as many more as fit (at most kMaxBufs).
__host__ __device__ inline AGeo make_ageo(const Dims &dm)
{
    const AGeo g0 = make_ageo_n(dm, 1);
    const int need = (int)((g0.off_phq + (size_t)128 * g0.FP * 2 - g0.off_R + g0.tileb - 1) / g0.tileb);
    int nb = need > 7 ? need : 7;
    AGeo g = make_ageo_n(dm, nb);
    while (nb < kMaxBufs) {
        const AGeo g2 = make_ageo_n(dm, nb + 1);
        if (g2.total > 227 * 1024) break;
        g = g2;
        ++nb;
    }
    return g;
}

// Thread 0 waits for an mbarrier phase (bounded); a timeout anywhere in the grid
// sets the device error word, after which every CTA stops waiting. CTA-uniform result.
__device__ __forceinline__ bool wait_mbar(uint64_t *mbar, uint32_t parity, int *okflag, int *err)
{
    if (threadIdx.x == 0) {
        const bool ok = umma::mbar_wait_abortable(mbar, parity, kWaitNs, err, ERR_TIMEOUT);
        if (!ok) raise_error(err, ERR_TIMEOUT);
        *okflag = ok ? 1 : 0;
    }
    __syncthreads();
    umma::fence_after_sync();
    return *okflag != 0;
}

// cp.async.wait_group with a run-time count (the ring depth is chosen at launch)
__device__ __forceinline__ void cp_wait_upto(int n)
{
    switch (n) {
    case 0: umma::cp_async_wait_n<0>(); break;
    case 1: umma::cp_async_wait_n<1>(); break;
    case 2: umma::cp_async_wait_n<2>(); break;
    case 3: umma::cp_async_wait_n<3>(); break;
    case 4: umma::cp_async_wait_n<4>(); break;
    case 5: umma::cp_async_wait_n<5>(); break;
    case 6: umma::cp_async_wait_n<6>(); break;
    case 7: umma::cp_async_wait_n<7>(); break;
    case 8: umma::cp_async_wait_n<8>(); break;
    case 9: umma::cp_async_wait_n<9>(); break;
    default: umma::cp_async_wait_all(); break;   // deeper rings wait for everything
    }
}

// MMA issue, one thread: D (+)= A[128 x K] * B, K = 16 * nks
// (descriptors are built once; a k-step only moves the start-address field, addr >> 4)
__device__ __forceinline__ uint32_t kstep_k(int ks, int R) { return (uint32_t)(((ks >> 2) * R * 128 + (ks & 3) * 32) >> 4); }
__device__ __forceinline__ void mma_kk(uint32_t dt, uint32_t a0, int ra, uint32_t b0, int rb, int nks,
                                       uint32_t idesc, bool acc)
{
    const uint64_t da = umma::kmajor_desc(a0, 0, ra), db = umma::kmajor_desc(b0, 0, rb);
    for (int ks = 0; ks < nks; ++ks)
        umma::mma_ss(dt, da + kstep_k(ks, ra), db + kstep_k(ks, rb), idesc, (acc || ks > 0) ? 1u : 0u);
}
__device__ __forceinline__ void mma_kn(uint32_t dt, uint32_t a0, int ra, uint32_t b0, int nb, int nks,
                                       uint32_t idesc, bool acc)
{
    const uint64_t da = umma::kmajor_desc(a0, 0, ra), db = umma::mnmajor_desc(b0, 0, nb);
    const uint32_t sb = (uint32_t)((2 * (nb >> 6) * 1024) >> 4);
    for (int ks = 0; ks < nks; ++ks)
        umma::mma_ss(dt, da + kstep_k(ks, ra), db + (uint64_t)(ks * sb), idesc, (acc || ks > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(Dims dm, DevState S, PrefillScratch P, AttnArgs a, KVSrc<bf16> src)
{
    if (cta_error_pending(S.err)) return;   // the chain of this call gave up: its logs are incomplete
    const AGeo g = make_ageo(dm);
    const int d = g.d, D = g.D, FP = g.FP, Dh = g.Dh, eta = dm.eta, lam = dm.lam, gq = dm.g;
    const int NK = g.NK, NV = g.NV, MS = g.MS;
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
    const float scale = rsqrtf((float)d);
    const int lgd = __ffs(d >> 3) - 1, lgf = __ffs(FP >> 3) - 1;   // 16-byte chunks per row

    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t bar_x, bar_s[2], bar_o[2];   // setup MMAs; scores of tile i (i & 1); PV of tile i
    __shared__ uint64_t bar_h;                        // the snapshot H' has landed (bulk copy)
    __shared__ uint32_t tslot;
    __shared__ int okflag;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *sQ = base, *sPr = base + g.off_P, *sR = base + g.off_R;
    uint8_t *sH = base + g.off_H, *sPhq = base + g.off_phq;
    TileMeta *meta = (TileMeta *)(base + g.off_meta);
    float *sS = (float *)(base + g.off_meta);        // s' during the setup
    float *red = (float *)(base + g.off_red);
    // ring buffers: keys of tile t in buffer 1 + t % NK; values of tile t in buffer
    // 1 + NK + t % NV, except slot NV - 1, which is buffer 0 (V_L of the setup)
    auto kbuf = [&](int t) { return sR + (size_t)(1 + t % NK) * g.tileb; };
    auto vbuf = [&](int t) {
        const int s = t % NV;
        return sR + (size_t)(s == NV - 1 ? 0 : 1 + NK + s) * g.tileb;
    };
    auto pbuf = [&](int i) { return sPr + (size_t)(i & 1) * 128 * KT * 2; };

    if (tid == 0) {
        umma::mbar_init(&bar_x, 1);
        umma::mbar_init(&bar_s[0], 1);
        umma::mbar_init(&bar_s[1], 1);
        umma::mbar_init(&bar_o[0], 2);   // PV (thread 0) and the row sums (thread 32) of tile i
        umma::mbar_init(&bar_o[1], 2);
        umma::mbar_init(&bar_h, 1);
    }
    if (warp == 0) umma::tmem_alloc(&tslot, g.ncols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tm = tslot;
    // O: columns [0, d), the sum of the weights: column d; score buffer b at tS0 + b * KT
    const uint32_t tO = tm, tS0 = tm + (uint32_t)g.NBa;
    uint8_t *sOnes = base + g.off_ones;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    uint32_t xph = 0;                                // phases of bar_x committed and waited for

    // ---- ones operand (row 0 of a K-major 16 x 64 tile), zero weight sums, stage Q, W^T
    //      (P region), H' and s'
    for (int e = tid; e < 16 * KT; e += kThreads) {
        const int rr = e / KT, k = e - rr * KT;
        *(bf16 *)(sOnes + umma::kmajor_offset(rr, k, 16)) = __float2bfloat16_rn(rr == 0 ? 1.f : 0.f);
    }
    if (half == 0) {
        float z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0.f;
        umma::tmem_st16(tO + lane_off + (uint32_t)d, z);
        umma::tmem_wait_st();
    }
    const bf16 *q = (const bf16 *)a.q;
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
        const bf16 *Wt = (const bf16 *)S.Wt + (dm.nW > 1 ? (size_t)hk * Dh * d : 0);
        for (int e = tid; e < (Dh << lgd); e += kThreads) {
            const int rr = e >> lgd, kc = e & ((1 << lgd) - 1);
            umma::cp_async16(sPr + umma::kmajor_offset(rr, kc * 8, Dh), Wt + (size_t)rr * d + kc * 8);
        }
    }
    // the snapshot: H' as an N-contiguous [FP][d] operand, stored in exactly that layout: one
    // bulk copy, in flight during Z and phi(Q) (waited for before the readout); then s' as
    // row 0 of a K-major 16 x FP operand
    const uint8_t *img = (const uint8_t *)P.snapImg + ((size_t)st * dm.mmax + ci) * (size_t)(FP * (d + 16) * 2);
    if (tid == 0) {
        umma::mbar_arrive_expect_tx(&bar_h, (uint32_t)(FP * d * 2));
        umma::bulk_g2s(sH, img, (uint32_t)(FP * d * 2), &bar_h);
    }
    for (int f = tid; f < FP; f += kThreads)
        sS[f] = __bfloat162float(*(const bf16 *)(img + (size_t)FP * d * 2 + umma::kmajor_offset(0, f, 16)));
    umma::cp_async_commit();
    umma::cp_async_wait_all();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();

    bool ok = true;
    // ---- Z = Q W on the tensor cores (into the score columns)
    if (tid == 0) {
        umma::fence_after_sync();
        mma_kk(tS0, umma::smem_u32(sQ), 128, umma::smem_u32(sPr), Dh, d / 16,
               umma::idesc_bf16(128, Dh, false, false), false);
        umma::mma_commit(&bar_x);
    }
    ok = wait_mbar(&bar_x, xph & 1u, &okflag, S.err);
    ++xph;

    // leaving pairs of this interval, [jL0, jL1): linear for a query once they left its
    // window, if they were folded
    const size_t lb = (size_t)st * dm.mmax + ci;
    const uint8_t *llf = P.logLf + lb * dm.Lmax;
    const long long jL0 = t0 - eta > 0 ? t0 - eta : 0;
    const long long jL1 = t1 - eta > jL0 ? t1 - eta : jL0;
    const int nLin = (int)(jL1 - jL0);
    const int nlch = (nLin + KT - 1) / KT;
    const bf16 *phiK = (const bf16 *)P.phiK + (size_t)st * (lam + dm.R + dm.Nmax) * D;
    // phi(K) rows of linear chunk c into the P region, its value rows into buffer 0
    auto issue_lin = [&](int c) {
        const long long j0 = jL0 + (long long)c * KT;
        const int nk = (int)min((long long)KT, jL1 - j0);
        for (int e = tid; e < (KT << lgf); e += kThreads) {
            const int j = e >> lgf, kc = e & ((1 << lgf) - 1);
            uint8_t *dst = sPr + umma::kmajor_offset(j, kc * 8, KT);
            if (j < nk && kc * 8 < D) umma::cp_async16(dst, phiK + (size_t)src.tok2vrow(j0 + j) * D + kc * 8);
            else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
        for (int e = tid; e < (KT << lgd); e += kThreads) {
            const int j = e >> lgd, kc = e & ((1 << lgd) - 1);
            uint8_t *dst = sR + umma::mnmajor_offset(j, kc * 8, d);
            if (j < nk) umma::cp_async16(dst, src.vrow(st, src.tok2vrow(j0 + j)) + kc * 8);
            else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
        umma::cp_async_commit();
    };
    if (ok && nLin > 0) issue_lin(0);   // W^T is dead: Z is complete

    // ---- phi(Q) = [softmax(Z), softmax(-Z)]: half 0 writes the first Dh features, half 1
    //      the last Dh, as bf16 into the K-major phi(Q) tile; l = phi(Q).s' from the same
    //      rounded features
    float lpart = 0.f;
    if (ok) {
        float zmax = -INFINITY, zmin = INFINITY;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS0 + lane_off + (uint32_t)c0, v);
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
            umma::tmem_ld16(tS0 + lane_off + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) ssum += half ? __expf(zmin - v[j]) : __expf(v[j] - zmax);
        }
        const float rs_ = 1.f / ssum;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(tS0 + lane_off + (uint32_t)c0, v);
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
                const int f0 = half * Dh + c0 + j;
                *(uint4 *)(sPhq + umma::kmajor_offset(r, f0, 128)) = pk;
                lpart += umma::bf16lo_to_f32(pk.x) * sS[f0] + umma::bf16hi_to_f32(pk.x) * sS[f0 + 1] +
                         umma::bf16lo_to_f32(pk.y) * sS[f0 + 2] + umma::bf16hi_to_f32(pk.y) * sS[f0 + 3] +
                         umma::bf16lo_to_f32(pk.z) * sS[f0 + 4] + umma::bf16hi_to_f32(pk.z) * sS[f0 + 5] +
                         umma::bf16lo_to_f32(pk.w) * sS[f0 + 6] + umma::bf16hi_to_f32(pk.w) * sS[f0 + 7];
            }
        }
        if (half == 1)
            for (int c = D; c < FP; c += 8)
                *(uint4 *)(sPhq + umma::kmajor_offset(r, c, 128)) = make_uint4(0, 0, 0, 0);
    }
    umma::cp_async_wait_all();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();

    // ---- O = phi(Q) H'; G = phi(Q) phi(K_L)^T of linear chunk 0 into the score columns
    const uint32_t id_g = umma::idesc_bf16(128, KT, false, false);
    const uint32_t id_one = umma::idesc_bf16(128, 16, false, false);   // P x ones: weight sums
    const uint32_t id_pv = umma::idesc_bf16(128, d, false, true);
    bool h_wt = false;   // thread 0: the snapshot copy was waited for
    if (ok) {
        if (tid == 0) {
            h_wt = umma::mbar_wait_abortable(&bar_h, 0, kWaitNs, S.err, ERR_TIMEOUT);
            if (!h_wt) raise_error(S.err, ERR_TIMEOUT);   // the MMA wait below gives up at once
            umma::fence_after_sync();
            const uint32_t a0 = umma::smem_u32(sPhq);
            mma_kn(tO, a0, 128, umma::smem_u32(sH), d, FP / 16, id_pv, false);
            if (nLin > 0) mma_kk(tS0, a0, 128, umma::smem_u32(sPr), KT, FP / 16, id_g, false);
            umma::mma_commit(&bar_x);
        }
        ok = wait_mbar(&bar_x, xph & 1u, &okflag, S.err);
        ++xph;
    }
    // ---- linear chunks: weights -G where the pair was folded but is still inside the
    //      window of the row's query; O += W V_L and l += sum W (the rounded weights),
    //      still at m = 0
    for (int c = 0; c < nlch && ok; ++c) {
        if (c > 0) {
            // the previous chunk's PV reads the P region and buffer 0
            if (tid == 0) umma::mma_commit(&bar_x);
            ok = wait_mbar(&bar_x, xph & 1u, &okflag, S.err);
            ++xph;
            if (!ok) break;
            issue_lin(c);
            umma::cp_async_wait_all();
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncthreads();
            if (tid == 0) {
                umma::fence_after_sync();
                mma_kk(tS0, umma::smem_u32(sPhq), 128, umma::smem_u32(sPr), KT, FP / 16, id_g, false);
                umma::mma_commit(&bar_x);
            }
            ok = wait_mbar(&bar_x, xph & 1u, &okflag, S.err);
            ++xph;
            if (!ok) break;
        }
        const long long j0 = jL0 + (long long)c * KT;
#pragma unroll
        for (int c0 = 0; c0 < 32; c0 += 16) {
            float gv[16];
            umma::tmem_ld16(tS0 + lane_off + (uint32_t)(half * 32 + c0), gv);
            umma::tmem_wait_ld();
            float w[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const long long j = j0 + half * 32 + c0 + jj;
                // folded, and still inside the window of the row's query: the snapshot holds
                // its linear term, the softmax attends it, so the linear term comes off
                const bool sub = row_ok && j < jL1 && j > p - eta && llf[(int)(j - (t0 - eta))] != 0;
                w[jj] = sub ? -gv[jj] : 0.f;
            }
#pragma unroll
            for (int h8 = 0; h8 < 16; h8 += 8) {
                uint4 pk;
                pk.x = umma::pack_bf16x2(w[h8 + 0], w[h8 + 1]);
                pk.y = umma::pack_bf16x2(w[h8 + 2], w[h8 + 3]);
                pk.z = umma::pack_bf16x2(w[h8 + 4], w[h8 + 5]);
                pk.w = umma::pack_bf16x2(w[h8 + 6], w[h8 + 7]);
                *(uint4 *)(pbuf(0) + umma::kmajor_offset(r, half * 32 + c0 + h8, 128)) = pk;
            }
        }
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            mma_kn(tO, umma::smem_u32(pbuf(0)), 128, umma::smem_u32(sR), d, KT / 16, id_pv, true);
            mma_kk(tO + (uint32_t)d, umma::smem_u32(pbuf(0)), 128, umma::smem_u32(sOnes), 16, KT / 16, id_one, true);
        }
    }

    // ---- softmax key tiles: the window [jL0, t1) first, then the interval's cached keys
    const int nK = P.logCount[lb];
    const int *ltok = P.logTok + lb * lam;
    const int *lvrow = P.logVrow + lb * lam;
    const int nband = (int)(t1 - jL0);
    const int ntb = (nband + KT - 1) / KT, ntc = (nK + KT - 1) / KT;
    const int n = ntb + ntc;
    // row addresses without per-row divisions: cache slot, window ring, or this call's input
    const size_t in_stride = (size_t)dm.Hkv * d;
    const size_t in_off = ((size_t)b * src.n * dm.Hkv + hk) * d;
    auto rowp = [&](const bf16 *cache, const bf16 *ring, const bf16 *in, int vr) -> const bf16 * {
        if (vr < lam) return cache + ((size_t)st * lam + vr) * d;
        if (vr < lam + dm.R) return ring + ((size_t)st * dm.R + (vr - lam)) * d;
        return in + in_off + (size_t)(vr - lam - dm.R) * in_stride;
    };
    // Tile metadata (token, value row, key class) moves through registers of threads
    // 0..63 (key = thread): loaded two tiles ahead of the key copies, stored to shared
    // memory one tile ahead, so no copy waits on a global load.
    auto meta_load = [&](int t, int &tok, int &vr, int &info) {
        tok = 0x7fffffff;
        vr = -1;
        info = INFO_SKIP;
        if (t >= n || tid >= KT) return;
        const int j = tid;
        if (t < ntb) {
            const long long kb = jL0 + (long long)t * KT;
            if (kb + j < t1) {
                const long long jj = kb + j;
                tok = (int)jj;
                vr = src.tok2vrow(jj);
                info = INFO_SOFT;
                if (jj < t1 - eta) info = llf[(int)(jj - (t0 - eta))] ? INFO_FOLDED : INFO_SKIP;
            }
        } else {
            const int kb = (t - ntb) * KT;
            if (kb + j < nK) {
                tok = ltok[kb + j];
                vr = lvrow[kb + j];
                info = INFO_SOFT;
            }
        }
    };
    auto meta_store = [&](int t, int tok, int vr, int info) {
        if (tid < KT) {   // warps 0 and 1, one key per thread
            TileMeta &M = meta[t % MS];
            M.tok[tid] = tok;
            M.vrow[tid] = vr;
            M.info[tid] = (unsigned char)info;
            const unsigned sk = __ballot_sync(0xffffffffu, info == INFO_SKIP);
            const unsigned fo = __ballot_sync(0xffffffffu, info == INFO_FOLDED);
            const int mx = __reduce_max_sync(0xffffffffu, info == INFO_SKIP ? (int)0x80000000 : tok);
            if (lane == 0) {
                M.skip32[warp] = sk;
                M.fold32[warp] = fo;
                M.maxtok32[warp] = mx;
            }
        }
    };
    // key rows of tile t into its K buffer (no commit); its metadata is in shared memory
    auto issue_k = [&](int t) {
        if (t >= n) return;
        const TileMeta &M = meta[t % MS];
        uint8_t *sK = kbuf(t);
        for (int e = tid; e < (KT << lgd); e += kThreads) {
            const int j = e >> lgd, kc = e & ((1 << lgd) - 1);
            uint8_t *dk = sK + umma::kmajor_offset(j, kc * 8, KT);
            const int vr = M.vrow[j];
            if (vr >= 0) umma::cp_async16(dk, rowp(src.KS, src.KR, src.kin, vr) + kc * 8);
            else *(uint4 *)dk = make_uint4(0, 0, 0, 0);
        }
    };
    // value rows of tile t (no commit)
    auto issue_v = [&](int t) {
        if (t >= n) return;
        const TileMeta &M = meta[t % MS];
        uint8_t *sV = vbuf(t);
        for (int e = tid; e < (KT << lgd); e += kThreads) {
            const int j = e >> lgd, kc = e & ((1 << lgd) - 1);
            uint8_t *dv = sV + umma::mnmajor_offset(j, kc * 8, d);
            const int vr = M.vrow[j];
            if (vr >= 0) umma::cp_async16(dv, rowp(src.VS, src.VR, src.vin, vr) + kc * 8);
            else *(uint4 *)dv = make_uint4(0, 0, 0, 0);
        }
    };
    const uint32_t id_s = umma::idesc_bf16(128, KT, false, false);
    auto issue_qk = [&](int t) {
        mma_kk(tS0 + (uint32_t)((t & 1) * KT), umma::smem_u32(sQ), 128, umma::smem_u32(kbuf(t)), KT, d / 16,
               id_s, false);
        umma::mma_commit(&bar_s[t & 1]);
    };
    // Ring bookkeeping: one cp.async group per tile in the prologue (keys 0..NK-1, then
    // values 0..NV-3), then one per iteration i (keys i+NK, values i+NV-2). At the end of
    // iteration i the keys of i+2 and the values of i are needed: all but the last NV-2
    // groups complete.
    int pf_tok, pf_vr, pf_info;   // metadata of the tile after the next one to be stored
    if (ok) {
        // H', phi(Q) and phi(K_L) are dead (their MMAs completed); V_L in buffer 0 and the
        // weights in P0 are still read by the last linear PV.
        // Metadata of tiles 0..NK (all loads in flight together), then tile NK+1 into registers.
        {
            int tk[kMaxPro], vk[kMaxPro], ik[kMaxPro];
#pragma unroll
            for (int t = 0; t < kMaxPro; ++t)
                if (t <= NK) meta_load(t, tk[t], vk[t], ik[t]);
#pragma unroll
            for (int t = 0; t < kMaxPro; ++t)
                if (t <= NK) meta_store(t, tk[t], vk[t], ik[t]);
            meta_load(NK + 1, pf_tok, pf_vr, pf_info);
        }
        __syncthreads();
        for (int t = 0; t < NK; ++t) {
            issue_k(t);
            umma::cp_async_commit();
        }
        for (int t = 0; t < NV - 2; ++t) {
            issue_v(t);
            umma::cp_async_commit();
        }
        cp_wait_upto(NK + NV - 4);   // keys of tiles 0 and 1
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            issue_qk(0);
            if (n > 1) issue_qk(1);
        }
    }

    float m = 0.f;
    int last_i = -1;                                  // last key tile whose MMAs were issued
    const int nch = (d + 16) / 16, split = nch / 2;   // O chunks (sums included) rescaled by half 0 / 1
    const float c1 = scale * 1.4426950408889634f;        // e^{x scale} = 2^{x c1}
    for (int i = 0; i < n && ok; ++i) {
        // scores of tile i; everything thread 0 issued before them (PV of tile i-2) is complete
        if (!(ok = wait_mbar(&bar_s[i & 1], (uint32_t)((i >> 1) & 1), &okflag, S.err))) break;
        if (i >= 2) {
            // and the row sums of tile i-2 (thread 32): their weight buffer is rewritten below
            if (lane == 0) {
                const bool okw = umma::mbar_wait_abortable(&bar_o[i & 1], (uint32_t)(((i - 2) >> 1) & 1), kWaitNs,
                                                           S.err, ERR_TIMEOUT);
                if (!okw) raise_error(S.err, ERR_TIMEOUT);
            }
            __syncwarp();
        }
        meta_store(i + NK + 1, pf_tok, pf_vr, pf_info);   // into the slot of tile i-1
        meta_load(i + NK + 2, pf_tok, pf_vr, pf_info);    // in flight during this tile
        issue_k(i + NK);        // into the buffer of tile i's keys
        issue_v(i + NV - 2);    // into the buffer of tile i-2's values
        umma::cp_async_commit();
        const TileMeta &M = meta[i % MS];

        // raw scores q.k (the 1/sqrt(d) scale is folded into the exponent)
        float sv[KT];
        {
            float v0[32], v1[32];
            umma::tmem_ld32(tS0 + (uint32_t)((i & 1) * KT) + lane_off, v0);
            umma::tmem_ld32(tS0 + (uint32_t)((i & 1) * KT) + lane_off + 32u, v1);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                sv[j] = v0[j];
                sv[32 + j] = v1[j];
            }
        }
        // live keys of this row (softmax keys it may see), one bit per key
        const unsigned long long skipm = (unsigned long long)M.skip32[0] | ((unsigned long long)M.skip32[1] << 32);
        unsigned long long live;
        if (i < ntb) {
            // window tile: token = kb + j; a folded pair is a softmax key only inside the window
            const long long kb = jL0 + (long long)i * KT;
            const unsigned long long foldm =
                (unsigned long long)M.fold32[0] | ((unsigned long long)M.fold32[1] << 32);
            live = ~skipm & prefix_mask(p - kb) & ~(foldm & prefix_mask(p - eta - kb));
        } else if ((long long)max(M.maxtok32[0], M.maxtok32[1]) <= p) {
            live = ~skipm;   // cached keys, all causal for this row
        } else {
            live = 0;
            for (int j = 0; j < KT; ++j)
                if (!((skipm >> j) & 1ull) && (long long)M.tok[j] <= p) live |= 1ull << j;
        }
        if (!row_ok) live = 0;
        const bool all_live = __all_sync(0xffffffffu, live == ~0ull);
        float tmax;
        {
            float t[32];
            if (all_live) {
#pragma unroll
                for (int j = 0; j < 32; ++j) t[j] = fmaxf(sv[j], sv[j + 32]);
            } else {
                const uint32_t lo = (uint32_t)live, hi = (uint32_t)(live >> 32);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    t[j] = fmaxf((lo >> j) & 1u ? sv[j] : -INFINITY, (hi >> j) & 1u ? sv[j + 32] : -INFINITY);
            }
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
            tmax = t[0];
        }
        tmax *= scale;
        // lazy rescaling: the shift m only moves when the row's maximum exceeds it by
        // more than kLazy (weights stay below e^kLazy; numerator and denominator share m)
        const bool grow_m = tmax > m + kLazy;
        if (__any_sync(0xffffffffu, grow_m)) {
            if (i > 0) {
                // PV of tile i-1 may still accumulate into O
                if (lane == 0) {
                    const bool okw = umma::mbar_wait_abortable(&bar_o[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1),
                                                               kWaitNs, S.err, ERR_TIMEOUT);
                    if (!okw) raise_error(S.err, ERR_TIMEOUT);
                }
                __syncwarp();
                umma::fence_after_sync();
            }
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
        const float mc = m * 1.4426950408889634f;
        const uint32_t w32 = (uint32_t)(live >> (half * 32));   // this half's keys
        uint8_t *sP = pbuf(i);
#pragma unroll
        for (int j0 = 0; j0 < 32; j0 += 8) {
            float pf[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int k = j0 + jj;
                const float s = half ? sv[32 + k] : sv[k];   // static indices keep sv in registers
                const float e = umma::ex2_approx(fmaf(s, c1, -mc));
                pf[jj] = all_live ? e : ((w32 >> k) & 1u ? e : 0.f);
            }
            uint4 pk;
            pk.x = umma::pack_bf16x2(pf[0], pf[1]);
            pk.y = umma::pack_bf16x2(pf[2], pf[3]);
            pk.z = umma::pack_bf16x2(pf[4], pf[5]);
            pk.w = umma::pack_bf16x2(pf[6], pf[7]);
            *(uint4 *)(sP + umma::kmajor_offset(r, half * 32 + j0, 128)) = pk;
        }
        // P of tile i is written; the keys of tile i+2 and the values of tile i have landed
        cp_wait_upto(NV - 2);
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            mma_kn(tO, umma::smem_u32(sP), 128, umma::smem_u32(vbuf(i)), d, KT / 16, id_pv, true);
            umma::mma_commit(&bar_o[i & 1]);
            if (i + 2 < n) issue_qk(i + 2);
        } else if (tid == 32) {
            // the row sums of the rounded weights the tensor core multiplied, into column d,
            // issued beside the PV by a second thread (other TMEM columns)
            umma::fence_after_sync();
            mma_kk(tO + (uint32_t)d, umma::smem_u32(sP), 128, umma::smem_u32(sOnes), 16, KT / 16, id_one, true);
            umma::mma_commit(&bar_o[i & 1]);
        }
        last_i = i;
    }

    // ---- drain: every MMA of this CTA is complete before its buffers and TMEM go away
    umma::cp_async_wait_all();
    if (tid == 0) {
        if (!h_wt) umma::mbar_wait(&bar_h, 0, kWaitNs);   // no copy outlives the CTA
        // the row sums of the last two tiles (thread 32's MMAs) are complete too
        for (int j = last_i - 1; j <= last_i; ++j)
            if (j >= 0) umma::mbar_wait(&bar_o[j & 1], (uint32_t)((j >> 1) & 1), kWaitNs);
        umma::mma_commit(&bar_x);
        const bool dok = umma::mbar_wait(&bar_x, xph & 1u, kWaitNs);
        if (!dok) raise_error(S.err, ERR_TIMEOUT);
        okflag = (ok && dok) ? 1 : 0;
    }
    __syncthreads();
    umma::fence_after_sync();
    ok = okflag != 0;

    if (ok) {
        // ---- normalise and store; half h writes value columns [h*d/2, (h+1)*d/2)
        if (half == 1) red[r] = lpart;
        __syncthreads();
        const float l = half == 0 ? lpart + red[r] : 0.f;
        __syncthreads();
        if (half == 0) red[r] = l;
        __syncthreads();
        float v[16];
        umma::tmem_ld16(tO + lane_off + (uint32_t)d, v);
        umma::tmem_wait_ld();
        const float den = red[r] + v[0] + dm.eps * __expf(-m);
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
