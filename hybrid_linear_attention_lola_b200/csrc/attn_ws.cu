// Warp-specialised tensor-core prefill output of a LoLA hybrid-attention layer
// for bfloat16 inputs: the same output as the single-tile kernel of attn_tc.cu
// (gist.science technical summary, "Inferentiestrategie": linear attention over
// the recurrent state + softmax attention over the sliding window and the
// sparse cache, one shared normaliser), with loads, tensor-core issue and the
// softmax running concurrently in separate warps, and two 128-row query tiles
// sharing every key and value tile.
//
// One CTA = one update interval of one (batch, kv-head) stream and nq (1 or 2)
// tiles of 128 query rows; row r of tile q is (position t0 + (tile*128 + r)/g,
// query head hk*g + r%g) and TMEM lane r of that tile's accumulators.
// Warps:  0-3 / 4-7  softmax of tile 0 / tile 1, one thread per row
//         8          rows 0-31 of every key tile; also Q, W^T, the snapshot halves and
//                    the band rows, and the tile metadata
//         9          rows 0-31 of every value tile
//         10         rows 32-63 of every key tile, then of the value tile
//         11         tensor-core issue (one thread)
// Gathered rows are latency-bound per SM (random 256-byte rows): three warps issuing
// copies keep more of them in flight than one per operand.
// Setup, all at shift m = 0; phi(Q) = [softmax(Z), softmax(-Z)], Z = Q W:
//   Z on the tensor cores; each softmax thread turns its row of Z into
//   e+ = exp(z - max z) and e- = exp(min z - z) and their sums s+, s-.
//   Two passes over the feature halves (e+ in pass 0, e- in pass 1) accumulate
//   O = phi(Q) H1, l = phi(Q).s1 (column d of O) and G = phi(Q) phi(K_L)^T; between
//   the passes O and G are multiplied by s-/s+, after them O by 1/s-, so each half
//   carries its own softmax normaliser. H1 is the interval's end state (every pair
//   the interval folds); the band weights -G/s- of folded leaving pairs still
//   inside a row's window go through one P V product per 64-key chunk.
// Main loop, per 64-key tile (window keys [t0 - eta, t1), then the interval's
// cached keys): S = Q K^T, P = e^{s - m} with a lazily moved shift m, O += P V; each
// softmax thread keeps the sum of its row's rounded weights. Key and value tiles
// stream through shared-memory rings: window tiles of this call's tokens as tiled
// TMA boxes, others (scattered cache rows) by 16-byte cp.async gathers.
// Finally out = O / (l + sum of weights + eps e^{-m}).
// Every wait is bounded; a timeout sets the device error word and every role
// leaves its loop, drains its copies and MMAs, and the CTA exits.
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {

namespace {

using bf16 = __nv_bfloat16;
constexpr int KT = 64;                       // keys per tile
constexpr int kWarpK = 8, kWarpV = 9, kWarpH = 10, kWarpM = 11;
constexpr int kThreads = 12 * 32;           // three warps per SM sub-partition (168 registers each)
constexpr float kLazy = 8.f;                 // shift slack of the lazy rescaling (natural log units)
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxRing = 8;                  // key (value) tile buffers, at most
constexpr int kMS = 8;                       // metadata slots
constexpr unsigned kFull = 0xffffffffu;
enum : int { INFO_SOFT = 0, INFO_FOLDED = 1, INFO_SKIP = 2 };

struct TileMeta {
    int tok[KT], vrow[KT];
    unsigned char info[KT];
    unsigned skip32[2], fold32[2];   // per 32 keys: never a softmax key here / a folded leaving pair
    int maxtok32[2];                 // per 32 keys: largest token of a key that is not skipped
    int tma;                         // 1: KT consecutive tokens of this call (tiled TMA boxes)
};

// Shared memory (offsets from a 1024-byte aligned base):
//   [Q tiles][metadata ring][X]
// X during the setup: [phi(Q) half of each tile (W^T first)][H' half][s' half]
//                     [phi(K_L) half per band chunk] ... [V_L per band chunk]
// X in the main loop: [P of each tile][key ring][value ring]
// V_L sits at or after the start of the value ring, which loads only once the
// band products are done; the key ring ends before V_L.
struct WGeo {
    int d, D, Dh, nq, nch, NBa, NK, NV;
    size_t qtile, ptile, tileb;
    size_t off_meta, off_X;
    size_t x_hh, x_sh, x_pk, x_vl, x_K, x_V;
    size_t total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WGeo make_wgeo_n(const Dims &dm, int nq, int NK, int NV)
{
    WGeo g{};
    g.d = dm.d;
    g.D = dm.D;
    g.Dh = dm.D / 2;
    g.nq = nq;
    g.nch = (dm.C + KT - 1) / KT;
    g.NBa = (dm.d + 16 + 31) / 32 * 32;
    g.NK = NK;
    g.NV = NV;
    g.qtile = (size_t)128 * dm.d * 2;
    g.ptile = (size_t)128 * KT * 2;
    g.tileb = (size_t)KT * dm.d * 2;
    g.off_meta = (size_t)nq * g.qtile;
    g.off_X = al(g.off_meta + (size_t)kMS * sizeof(TileMeta), 1024);
    const size_t pq = (size_t)nq * 128 * g.Dh * 2, wt = (size_t)g.Dh * dm.d * 2;
    g.x_hh = al(pq > wt ? pq : wt, 1024);
    g.x_sh = g.x_hh + al((size_t)g.Dh * dm.d * 2, 1024);
    g.x_pk = g.x_sh + al((size_t)16 * g.Dh * 2, 1024);
    const size_t pk_end = g.x_pk + (size_t)g.nch * KT * g.Dh * 2;
    g.x_K = (size_t)nq * g.ptile;
    g.x_V = g.x_K + (size_t)NK * g.tileb;
    const size_t main_end = g.x_V + (size_t)NV * g.tileb;
    g.x_vl = al(pk_end > g.x_V ? pk_end : g.x_V, 1024);
    const size_t setup_end = g.x_vl + (size_t)g.nch * g.tileb;
    g.total = g.off_X + (setup_end > main_end ? setup_end : main_end) + 1024;
    return g;
}

// Two query tiles per CTA (the kernel exists to share every key and value tile between
// them; with one tile per CTA the single-tile kernel, whose eight warps all gather and
// all run the softmax, is faster), then the deepest rings that fit (keys one deeper
// than values). Other shapes take the single-tile kernel.
inline bool make_wgeo(const Dims &dm, WGeo *out)
{
    if (dm.dtype != 1 || !dm.tc_chain || dm.d % 64 != 0 || (dm.D / 2) % 64 != 0 || 128 % dm.g != 0 || dm.lam <= 0)
        return false;
    const int tpi = (dm.C * dm.g + 127) / 128;
    const int nch = (dm.C + KT - 1) / KT;
    const int NBa = (dm.d + 16 + 31) / 32 * 32;
    for (int nq = tpi >= 2 ? 2 : 0; nq >= 2; --nq) {
        if (nq * NBa + nq * nch * KT > 512 || nq * (dm.D / 2) > 512) continue;
        for (int s = 2 * kMaxRing; s >= 4; --s) {
            const WGeo g = make_wgeo_n(dm, nq, (s + 1) / 2, s / 2);
            if (g.total <= 227 * 1024 - 2048) {   // room for the static barriers
                *out = g;
                return true;
            }
        }
    }
    return false;
}

// bits 0..x set (none for x < 0, all for x >= 63)
__device__ __forceinline__ unsigned long long prefix_mask(long long x)
{
    return x < 0 ? 0ull : x >= 63 ? ~0ull : (2ull << x) - 1ull;
}

// MMA issue, one thread: D (+)= A[128 x K] * B, K = 16 * nks (the descriptors are built
// once; a k-step only moves the start address field, addr >> 4)
__device__ __forceinline__ uint32_t kstep_k(int ks, int R) { return (uint32_t)(((ks >> 2) * R * 128 + (ks & 3) * 32) >> 4); }
__device__ __forceinline__ void mma_kk(uint32_t dt, uint32_t a0, int ra, uint32_t b0, int rb, int nks,
                                       uint32_t idesc, bool acc)
{
    const uint64_t da = umma::kmajor_desc(a0, 0, ra), db = umma::kmajor_desc(b0, 0, rb);
    for (int ks = 0; ks < nks; ++ks)
        umma::mma_ss(dt, da + kstep_k(ks, ra), db + kstep_k(ks, rb), idesc, (acc || ks > 0) ? 1u : 0u);
}
// B N-contiguous in the [k/8][n/64][k%8][128 B] layout (the snapshot image)
__device__ __forceinline__ void mma_kn(uint32_t dt, uint32_t a0, int ra, uint32_t b0, int nb, int nks,
                                       uint32_t idesc, bool acc)
{
    const uint64_t da = umma::kmajor_desc(a0, 0, ra), db = umma::mnmajor_desc(b0, 0, nb);
    const uint32_t sb = (uint32_t)((2 * (nb >> 6) * 1024) >> 4);
    for (int ks = 0; ks < nks; ++ks)
        umma::mma_ss(dt, da + kstep_k(ks, ra), db + (uint64_t)(ks * sb), idesc, (acc || ks > 0) ? 1u : 0u);
}
// O += P V: P is a K-major 128 x 64 weight tile, V a 64-key value tile in the
// [n/64][key][128 B] layout (N-contiguous; 64-column blocks KT * 128 bytes apart,
// 8-key groups 1024 bytes apart). The row sums of P are kept by the softmax threads
// (a 128 x 16 MMA against a ones operand costs as much issue time as a 128 x 64 one).
__device__ __forceinline__ void mma_pv(uint32_t dt, uint32_t p0, uint32_t v0, int d)
{
    const uint64_t da = umma::kmajor_desc(p0, 0, 128);
    const uint64_t db = umma::make_desc(v0, (uint32_t)(KT * 128), 1024);
    const uint32_t id_pv = umma::idesc_bf16(128, d, false, true);
#pragma unroll
    for (int ks = 0; ks < KT / 16; ++ks)
        umma::mma_ss(dt, da + kstep_k(ks, 128), db + (uint64_t)((ks * 2048) >> 4), id_pv, 1u);
}

// sum of the eight bf16 values of four packed pairs
__device__ __forceinline__ float sum_bf16x8(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return (umma::bf16lo_to_f32(a) + umma::bf16hi_to_f32(a)) + (umma::bf16lo_to_f32(b) + umma::bf16hi_to_f32(b)) +
           (umma::bf16lo_to_f32(c) + umma::bf16hi_to_f32(c)) + (umma::bf16lo_to_f32(d) + umma::bf16hi_to_f32(d));
}

// fp32 x scalar over n columns (n a multiple of 16) of this warp's 32 TMEM lanes
__device__ __forceinline__ void tmem_scale(uint32_t taddr, int n, float f)
{
    for (int c0 = 0; c0 < n; c0 += 16) {
        float v[16];
        umma::tmem_ld16(taddr + (uint32_t)c0, v);
        umma::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] *= f;
        umma::tmem_st16(taddr + (uint32_t)c0, v);
    }
}

// Waits for an mbarrier phase (bounded); a timeout sets the error word, after which
// later waits give up at once.
__device__ __forceinline__ bool waitb(uint64_t *bar, uint32_t par, int *err)
{
    const bool ok = umma::mbar_wait_abortable(bar, par, kWaitNs, err, ERR_TIMEOUT);
    if (!ok) raise_error(err, ERR_TIMEOUT);
    return ok;
}
// warp-uniform wait: lane 0 waits, the warp takes its result (and its view of memory)
__device__ __forceinline__ bool waitw(uint64_t *bar, uint32_t par, int *err)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = waitb(bar, par, err) ? 1 : 0;
    ok = __shfl_sync(kFull, ok, 0);
    __syncwarp();
    return ok != 0;
}
__device__ __forceinline__ uint4 u4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return make_uint4(a, b, c, d);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_ws_kernel(Dims dm, DevState S, PrefillScratch P, AttnArgs a, KVSrc<bf16> src, WGeo G,
                   const __grid_constant__ AttnMaps maps)
{
    if (cta_error_pending(S.err)) return;   // the chain of this call gave up: its logs are incomplete
    const int d = G.d, D = G.D, Dh = G.Dh, NK = G.NK, NV = G.NV;
    const int eta = dm.eta, lam = dm.lam, gq = dm.g;
    const int tpi = (dm.C * gq + 127) / 128;
    const int cpi = (tpi + G.nq - 1) / G.nq;
    const int ci = a.ci0 + blockIdx.x / cpi;
    const int tile0 = (blockIdx.x % cpi) * G.nq;
    const int nqe = min(G.nq, tpi - tile0);
    const int st = blockIdx.y, b = st / dm.Hkv, hk = st % dm.Hkv;
    const long long t0 = a.pos0 + (long long)ci * dm.C, t1 = t0 + dm.C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rows_total = dm.C * gq;
    int *err = S.err;

    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t bq, bh[2], bz, bphq[2], bpass[2], bvl, bband, bdone, bdrain;
    __shared__ uint64_t kfull[kMaxRing], kempty[kMaxRing], vfull[kMaxRing], vempty[kMaxRing];
    __shared__ uint64_t mfull[kMS], mempty[kMS];
    __shared__ uint64_t sfull[2], sfree[2], pfull[2], pfree[2], bread[2];
    __shared__ uint32_t tslot;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *sX = base + G.off_X;
    TileMeta *meta = (TileMeta *)(base + G.off_meta);
    uint8_t *sHH = sX + G.x_hh, *sSH = sX + G.x_sh, *sPK = sX + G.x_pk, *sVL = sX + G.x_vl;
    auto sQ = [&](int q) { return base + (size_t)q * G.qtile; };
    auto sP = [&](int q) { return sX + (size_t)q * G.ptile; };
    auto pq = [&](int q) { return sX + (size_t)q * 128 * Dh * 2; };
    auto kbuf = [&](int t) { return sX + G.x_K + (size_t)(t % NK) * G.tileb; };
    auto vbuf = [&](int t) { return sX + G.x_V + (size_t)(t % NV) * G.tileb; };

    // the interval: leaving pairs [jL0, jL1), band keys [jL0, t1), the cached keys
    const size_t lb = (size_t)st * dm.mmax + ci;
    const uint8_t *llf = P.logLf + lb * dm.Lmax;
    const long long jL0 = t0 - eta > 0 ? t0 - eta : 0;
    const long long jL1 = t1 - eta > jL0 ? t1 - eta : jL0;
    const int nLin = (int)(jL1 - jL0);
    const int nchi = (nLin + KT - 1) / KT;
    const int nK = P.logCount[lb];
    const int *ltok = P.logTok + lb * lam;
    const int *lvrow = P.logVrow + lb * lam;
    const int nband = (int)(t1 - jL0);
    const int ntb = (nband + KT - 1) / KT, ntc = (nK + KT - 1) / KT;
    const int n = ntb + ntc;
    const long long zrow0 = (long long)b * a.n_call - a.pos0;   // TMA token coordinate of token t: zrow0 + t

    if (tid == 0) {
        umma::mbar_init(&bq, 1);
        umma::mbar_init(&bh[0], 1);
        umma::mbar_init(&bh[1], 1);
        umma::mbar_init(&bz, 1);
        umma::mbar_init(&bphq[0], 4 * nqe);
        umma::mbar_init(&bphq[1], 4 * nqe);
        umma::mbar_init(&bpass[0], 1);
        umma::mbar_init(&bpass[1], 1);
        umma::mbar_init(&bvl, 1);
        umma::mbar_init(&bband, 1);
        umma::mbar_init(&bdone, 1);
        umma::mbar_init(&bdrain, 1);
        for (int i = 0; i < NK; ++i) {
            umma::mbar_init(&kfull[i], 64);   // the lanes of the two warps loading it, once their copies landed
            umma::mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            umma::mbar_init(&vfull[i], 64);
            umma::mbar_init(&vempty[i], 1);
        }
        for (int i = 0; i < kMS; ++i) {
            umma::mbar_init(&mfull[i], 1);
            umma::mbar_init(&mempty[i], 2 + 4 * nqe);   // its readers: warps 9, 10 and the softmax warps
        }
        for (int q = 0; q < 2; ++q) {
            umma::mbar_init(&sfull[q], 1);
            umma::mbar_init(&sfree[q], 4);
            umma::mbar_init(&pfull[q], 4);
            umma::mbar_init(&pfree[q], 1);
            umma::mbar_init(&bread[q], 4);
        }
    }
    if (warp == kWarpM) umma::tmem_alloc(&tslot, 512);
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tm = tslot;
    // TMEM: O of tile q (d columns + the linear denominator in column d) at q * NBa; score / band buffer
    // of tile q and chunk c after them; Z of tile q at q * Dh (setup only)
    auto tO = [&](int q) { return tm + (uint32_t)(q * G.NBa); };
    auto tG = [&](int q, int c) { return tm + (uint32_t)(G.nq * G.NBa + (c * G.nq + q) * KT); };
    auto tZ = [&](int q) { return tm + (uint32_t)(q * Dh); };

    // virtual row -> address of its key / value row
    const size_t in_stride = (size_t)dm.Hkv * d;
    const size_t in_off = ((size_t)b * src.n * dm.Hkv + hk) * d;
    auto rowp = [&](const bf16 *cache, const bf16 *ring, const bf16 *in, int vr) -> const bf16 * {
        if (vr < lam) return cache + ((size_t)st * lam + vr) * d;
        if (vr < lam + dm.R) return ring + ((size_t)st * dm.R + (vr - lam)) * d;
        return in + in_off + (size_t)(vr - lam - dm.R) * in_stride;
    };
    // 16-byte copies of the 64 rows of a tile (key or value; both in the K-major layout of
    // a 64-row operand, which is also the N-contiguous layout mma_pv reads); a row with no
    // virtual row is zero-filled by the copy itself, so that every byte of the tile lands
    // through the copies the lane's mbarrier arrival waits for
    auto gather = [&](uint8_t *dst, const TileMeta &M, const bf16 *cache, const bf16 *ring, const bf16 *in,
                      int part) {
        const int cpr = d >> 3, rpi = 32 / cpr;
        const int kc = lane % cpr;
        const int j1 = (part + 1) * (KT / 2);
        for (int j = part * (KT / 2) + lane / cpr; j < j1; j += rpi) {
            const int vr = M.vrow[j];
            uint8_t *dk = dst + umma::kmajor_offset(j, kc * 8, KT);
            if (vr >= 0) umma::cp_async16(dk, rowp(cache, ring, in, vr) + kc * 8);
            else umma::cp_async16_zfill(dk, cache, 0u);
        }
    };

    if (warp >= kWarpK && warp < kWarpM) {
        // ================= load warps =================
        const bool kl = warp == kWarpK;   // key lead: setup loads and the tile metadata
        bool ok = true;
        bool issued_h1 = false;
        const long long nvr = (long long)lam + dm.R + dm.Nmax;
        const bf16 *phiK_st = (const bf16 *)P.phiK + (size_t)st * nvr * D;
        auto chunk_tma = [&](int c) { return jL0 + (long long)c * KT >= a.pos0; };
        if (kl) {
            // ---- Q tiles and W^T (into the phi(Q) slot)
            if (lane == 0) {
                umma::mbar_arrive_expect_tx(&bq, (uint32_t)(nqe * G.qtile + (size_t)Dh * d * 2));
                for (int q = 0; q < nqe; ++q) {
                    const int z = (int)(zrow0 + t0) + (tile0 + q) * (128 / gq);
                    for (int a2 = 0; a2 < d / 64; ++a2)
                        umma::tma_load_3d(sQ(q) + (size_t)a2 * 128 * 128, &maps.q, a2 * 64, hk * gq, z, &bq);
                }
                const bf16 *wt = (const bf16 *)S.WtImg + (dm.nW > 1 ? (size_t)hk * Dh * d : 0);
                umma::bulk_g2s(pq(0), wt, (uint32_t)(Dh * d * 2), &bq);
            }
            // ---- pass h: H' rows [h Dh, (h+1) Dh) (contiguous in the image), the s' blocks
            //      of the half, phi(K_L) of every band chunk (features of the half)
            const uint8_t *img = (const uint8_t *)P.snapImg + lb * (size_t)(D * (d + 16) * 2);
            auto load_pass = [&](int h) {
                bool any = false;
                for (int c = 0; c < nchi; ++c) {
                    if (chunk_tma(c)) continue;
                    any = true;   // rows of the window ring: 16-byte copies
                    const long long j0 = jL0 + (long long)c * KT;
                    uint8_t *dst0 = sPK + (size_t)c * KT * Dh * 2;
                    const int cpr = Dh >> 3;
                    for (int e = lane; e < KT * cpr; e += 32) {
                        const int j = e / cpr, kc = e - j * cpr;
                        uint8_t *dst = dst0 + umma::kmajor_offset(j, kc * 8, KT);
                        if (j0 + j < t1)
                            umma::cp_async16(dst, phiK_st + (size_t)src.tok2vrow(j0 + j) * D + h * Dh + kc * 8);
                        else
                            *(uint4 *)dst = u4(0, 0, 0, 0);
                    }
                }
                if (any) {
                    umma::cp_async_commit();
                    umma::cp_async_wait_all();
                    umma::fence_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    uint32_t bytes = (uint32_t)(Dh * d * 2 + Dh * 32);
                    for (int c = 0; c < nchi; ++c)
                        if (chunk_tma(c)) bytes += (uint32_t)(KT * Dh * 2);
                    umma::mbar_arrive_expect_tx(&bh[h], bytes);
                    umma::bulk_g2s(sHH, img + (size_t)h * Dh * d * 2, (uint32_t)(Dh * d * 2), &bh[h]);
                    umma::bulk_g2s(sSH, img + (size_t)D * d * 2 + (size_t)h * Dh * 32, (uint32_t)(Dh * 32), &bh[h]);
                    for (int c = 0; c < nchi; ++c) {
                        if (!chunk_tma(c)) continue;
                        const int y = (int)((long long)st * nvr + src.tok2vrow(jL0 + (long long)c * KT));
                        for (int a2 = 0; a2 < Dh / 64; ++a2)
                            umma::tma_load_2d(sPK + (size_t)c * KT * Dh * 2 + (size_t)a2 * KT * 128, &maps.phik,
                                              h * Dh + a2 * 64, y, &bh[h]);
                    }
                }
            };
            load_pass(0);
            // ---- V_L of every band chunk
            {
                bool any = false;
                for (int c = 0; c < nchi; ++c) {
                    if (chunk_tma(c)) continue;
                    any = true;
                    const long long j0 = jL0 + (long long)c * KT;
                    const int cpr = d >> 3;
                    for (int e = lane; e < KT * cpr; e += 32) {
                        const int j = e / cpr, kc = e - j * cpr;
                        uint8_t *dst = sVL + (size_t)c * G.tileb + umma::kmajor_offset(j, kc * 8, KT);
                        if (j0 + j < t1) umma::cp_async16(dst, src.vrow(st, src.tok2vrow(j0 + j)) + kc * 8);
                        else *(uint4 *)dst = u4(0, 0, 0, 0);
                    }
                }
                if (any) {
                    umma::cp_async_commit();
                    umma::cp_async_wait_all();
                    umma::fence_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    uint32_t bytes = 0;
                    for (int c = 0; c < nchi; ++c)
                        if (chunk_tma(c)) bytes += (uint32_t)G.tileb;
                    umma::mbar_arrive_expect_tx(&bvl, bytes);
                    for (int c = 0; c < nchi; ++c) {
                        if (!chunk_tma(c)) continue;
                        const int z = (int)(zrow0 + jL0 + (long long)c * KT);
                        for (int a2 = 0; a2 < d / 64; ++a2)
                            umma::tma_load_3d(sVL + (size_t)c * G.tileb + (size_t)a2 * KT * 128, &maps.v, a2 * 64, hk,
                                              z, &bvl);
                    }
                }
            }
            if ((ok = waitw(&bpass[0], 0, err))) {
                load_pass(1);
                issued_h1 = true;
                ok = waitw(&bpass[1], 0, err);   // the setup region is free for the key ring
            }
        } else if (warp == kWarpH) {
            ok = waitw(&bpass[1], 0, err);       // the setup region is free for the key ring
        } else {
            ok = waitw(&bband, 0, err);          // V_L has been read: the value ring may load
        }
        bool vfree = warp == kWarpV;             // the helper waits for the band before its first value rows

        // ---- the rings: tile t into buffer t % NK (keys) / t % NV (values). The full barrier
        //      of a buffer counts the lanes of the two warps that load it: after a gather
        //      every lane arrives once its own copies landed (the hardware does the arrival);
        //      for a TMA tile the lead's lane 0 arrives with the byte count and the others
        //      arrive at once. The load warps never wait for their copies.
        // metadata of tile t, key j: token, virtual row, key class
        auto fetch = [&](int t, int j, int &tok, int &vr, int &info) {
            tok = 0x7fffffff;
            vr = -1;
            info = INFO_SKIP;
            if (t >= n) return;
            if (t < ntb) {
                const long long jj = jL0 + (long long)t * KT + j;
                if (jj < t1) {
                    tok = (int)jj;
                    vr = src.tok2vrow(jj);
                    info = INFO_SOFT;
                    if (jj < t1 - eta) info = llf[(int)(jj - (t0 - eta))] ? INFO_FOLDED : INFO_SKIP;
                }
            } else {
                const int kc = (t - ntb) * KT + j;
                if (kc < nK) {
                    tok = ltok[kc];
                    vr = lvrow[kc];
                    info = INFO_SOFT;
                }
            }
        };
        // one operand's rows of tile t: keys (isK) or values, rows [32 part, 32 part + 32)
        auto load_part = [&](int t, const TileMeta &M, bool isK, int part) -> bool {
            const int nbuf = isK ? NK : NV, slot = t % nbuf;
            uint64_t *fullb = isK ? &kfull[slot] : &vfull[slot];
            if (t >= nbuf && !waitw(isK ? &kempty[slot] : &vempty[slot], (uint32_t)(((t / nbuf) - 1) & 1), err))
                return false;
            uint8_t *dst = isK ? kbuf(t) : vbuf(t);
            if (M.tma) {
                if (part == 0 && lane == 0) {
                    const long long kb = jL0 + (long long)t * KT;
                    umma::mbar_arrive_expect_tx(fullb, (uint32_t)G.tileb);
                    for (int a2 = 0; a2 < d / 64; ++a2)
                        umma::tma_load_3d(dst + (size_t)a2 * KT * 128, isK ? &maps.k : &maps.v, a2 * 64, hk,
                                          (int)(zrow0 + kb), fullb);
                } else {
                    umma::mbar_arrive(fullb);
                }
            } else {
                if (isK) gather(dst, M, src.KS, src.KR, src.kin, part);
                else gather(dst, M, src.VS, src.VR, src.vin, part);
                umma::cp_async_arrive_noinc(fullb);
            }
            return true;
        };
        int ftok[2], fvr[2], finfo[2];   // tile t's metadata, fetched during tile t - 1
        if (kl)
            for (int h2 = 0; h2 < 2; ++h2) fetch(0, lane + 32 * h2, ftok[h2], fvr[h2], finfo[h2]);
        int t_iss = 0;
        for (int t = 0; t < n && ok; ++t) {
            const int msl = t % kMS;
            TileMeta &M = meta[msl];
            if (kl) {
                if (t >= kMS && !(ok = waitw(&mempty[msl], (uint32_t)(((t / kMS) - 1) & 1), err))) break;
                const bool win = t < ntb;
                const bool tma = win && jL0 + (long long)t * KT >= a.pos0;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int j = lane + 32 * h2;
                    const int tok = ftok[h2], info = finfo[h2];
                    M.tok[j] = tok;
                    M.vrow[j] = fvr[h2];
                    M.info[j] = (unsigned char)info;
                    const unsigned sk = __ballot_sync(kFull, info == INFO_SKIP);
                    const unsigned fo = __ballot_sync(kFull, info == INFO_FOLDED);
                    const int mx = __reduce_max_sync(kFull, info == INFO_SKIP ? (int)0x80000000 : tok);
                    if (lane == 0) {
                        M.skip32[h2] = sk;
                        M.fold32[h2] = fo;
                        M.maxtok32[h2] = mx;
                    }
                }
                if (lane == 0) M.tma = tma ? 1 : 0;
                __syncwarp();
                if (lane == 0) umma::mbar_arrive(&mfull[msl]);
                // the next tile's metadata loads are in flight while this tile's rows go out
                for (int h2 = 0; h2 < 2; ++h2) fetch(t + 1, lane + 32 * h2, ftok[h2], fvr[h2], finfo[h2]);
                if (!(ok = load_part(t, M, true, 0))) break;
            } else {
                if (!(ok = waitw(&mfull[msl], (uint32_t)((t / kMS) & 1), err))) break;
                if (warp == kWarpH && !(ok = load_part(t, M, true, 1))) break;
                if (!vfree) {
                    if (!(ok = waitw(&bband, 0, err))) break;
                    vfree = true;
                }
                if (!(ok = load_part(t, M, false, warp == kWarpV ? 0 : 1))) break;
                __syncwarp();
                if (lane == 0) umma::mbar_arrive(&mempty[msl]);   // done with the metadata
            }
            ++t_iss;
        }
        umma::cp_async_wait_all();
        if (lane == 0) {
            // no copy or arrival outlives the CTA (the consumer waited for all of these unless
            // a wait gave up), nor the setup copies
            const bool doK = warp != kWarpV, doV = warp != kWarpK;
            for (int t = t_iss - NK > 0 ? t_iss - NK : 0; doK && t < t_iss; ++t)
                umma::mbar_wait(&kfull[t % NK], (uint32_t)((t / NK) & 1), kWaitNs);
            for (int t = t_iss - NV > 0 ? t_iss - NV : 0; doV && t < t_iss; ++t)
                umma::mbar_wait(&vfull[t % NV], (uint32_t)((t / NV) & 1), kWaitNs);
            if (kl) {
                umma::mbar_wait(&bq, 0, kWaitNs);
                umma::mbar_wait(&bh[0], 0, kWaitNs);
                if (issued_h1) umma::mbar_wait(&bh[1], 0, kWaitNs);
                umma::mbar_wait(&bvl, 0, kWaitNs);
            }
        }
        __syncwarp();
    } else if (warp == kWarpM) {
        // ================= tensor-core issue (lane 0) =================
        if (lane == 0) {
            bool ok = true;
            int u = 0;   // uses of the weight buffers (band chunks, then key tiles)
            // Z = Q W
            if ((ok = waitb(&bq, 0, err))) {
                umma::fence_after_sync();
                for (int q = 0; q < nqe; ++q)
                    mma_kk(tZ(q), umma::smem_u32(sQ(q)), 128, umma::smem_u32(pq(0)), Dh, d / 16,
                           umma::idesc_bf16(128, Dh, false, false), false);
                umma::mma_commit(&bz);
            }
            // the two feature passes: O, the sums column and G
            for (int h = 0; h < 2 && ok; ++h) {
                if (!(ok = waitb(&bphq[h], 0, err) && waitb(&bh[h], 0, err))) break;
                umma::fence_after_sync();
                for (int q = 0; q < nqe; ++q) {
                    const uint32_t a0 = umma::smem_u32(pq(q));
                    mma_kn(tO(q), a0, 128, umma::smem_u32(sHH), d, Dh / 16, umma::idesc_bf16(128, d, false, true), h > 0);
                    mma_kk(tO(q) + (uint32_t)d, a0, 128, umma::smem_u32(sSH), 16, Dh / 16,
                           umma::idesc_bf16(128, 16, false, false), h > 0);
                    for (int c = 0; c < nchi; ++c)
                        mma_kk(tG(q, c), a0, 128, umma::smem_u32(sPK + (size_t)c * KT * Dh * 2), KT, Dh / 16,
                               umma::idesc_bf16(128, KT, false, false), h > 0);
                }
                umma::mma_commit(&bpass[h]);
            }
            // band chunks: O += W V_L
            for (int c = 0; c < nchi && ok; ++c) {
                if (c == 0 && !(ok = waitb(&bvl, 0, err))) break;
                for (int q = 0; q < nqe && ok; ++q) {
                    if (!(ok = waitb(&pfull[q], (uint32_t)(u & 1), err))) break;
                    umma::fence_after_sync();
                    mma_pv(tO(q), umma::smem_u32(sP(q)), umma::smem_u32(sVL + (size_t)c * G.tileb), d);
                    umma::mma_commit(&pfree[q]);
                }
                ++u;
            }
            umma::mma_commit(&bband);   // V_L is free once these products are done
            // key tiles, an event loop over the two query tiles: S_q(i) = Q_q K(i)^T goes out
            // once the key tile has landed and tile q's softmax has read S_q(i - 1); P_q V(j)
            // once the value tile has landed and tile q's weights are written. The two tiles
            // never wait for each other; a key (value) buffer is released after both tiles'
            // products that read it.
            const uint32_t id_s = umma::idesc_bf16(128, KT, false, false);
            int qk[2] = {0, 0}, pv[2] = {0, 0};
            for (int q = nqe; q < 2; ++q) qk[q] = pv[q] = n;   // no such tile
            uint64_t t_last = 0;
            unsigned idle = 0;
            while (ok && (pv[0] < n || pv[1] < n)) {
                bool prog = false;
                for (int q = 0; q < nqe; ++q) {
                    const int i = qk[q];
                    if (i >= n) continue;
                    if (!umma::mbar_test(&kfull[i % NK], (uint32_t)((i / NK) & 1))) continue;
                    if (!(i == 0 ? umma::mbar_test(&bread[q], 0) : umma::mbar_test(&sfree[q], (uint32_t)((i - 1) & 1))))
                        continue;
                    umma::fence_async_smem();   // the gathered rows (generic-proxy copies) to the tensor core
                    umma::fence_after_sync();
                    mma_kk(tG(q, 0), umma::smem_u32(sQ(q)), 128, umma::smem_u32(kbuf(i)), KT, d / 16, id_s, false);
                    umma::mma_commit(&sfull[q]);
                    qk[q] = i + 1;
                    if (qk[0] > i && qk[1] > i) umma::mma_commit(&kempty[i % NK]);
                    prog = true;
                }
                for (int q = 0; q < nqe; ++q) {
                    const int j = pv[q];
                    if (j >= qk[q]) continue;
                    if (!umma::mbar_test(&vfull[j % NV], (uint32_t)((j / NV) & 1))) continue;
                    if (!umma::mbar_test(&pfull[q], (uint32_t)((nchi + j) & 1))) continue;
                    umma::fence_async_smem();
                    umma::fence_after_sync();
                    mma_pv(tO(q), umma::smem_u32(sP(q)), umma::smem_u32(vbuf(j)), d);
                    umma::mma_commit(&pfree[q]);
                    pv[q] = j + 1;
                    if (pv[0] > j && pv[1] > j) umma::mma_commit(&vempty[j % NV]);
                    prog = true;
                }
                if (prog) {
                    idle = 0;
                    continue;
                }
                // nothing ready: back off; give up after kWaitNs without progress, or at once
                // once another thread has recorded an error
                if (idle++ == 0) t_last = umma::globaltimer_ns();
                __nanosleep(32);
                if ((idle & 255u) == 0) {
                    if ((*(const volatile int *)err & ERR_TIMEOUT) != 0) ok = false;
                    else if (umma::globaltimer_ns() - t_last > kWaitNs) {
                        raise_error(err, ERR_TIMEOUT);
                        ok = false;
                    }
                }
            }
            umma::mma_commit(&bdone);
            // every MMA of this CTA is complete before TMEM and the buffers go away
            umma::mma_commit(&bdrain);
            if (!umma::mbar_wait(&bdrain, 0, kWaitNs)) raise_error(err, ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < 4 * nqe) {
        // ================= softmax of tile q, one thread per row =================
        const int q = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lo = (uint32_t)(wq * 32) << 16;
        const int grow = (tile0 + q) * 128 + r;
        const bool row_ok = grow < rows_total;
        const long long p = t0 + grow / gq;
        uint8_t *myP = sP(q);
        bool ok = waitw(&bz, 0, err);
        float sp = 1.f, sn = 1.f;
        uint32_t E1[64];   // e- features of the row (bf16 pairs), held for pass 1
        if (ok) {
            umma::fence_after_sync();
            float zmax = -INFINITY, zmin = INFINITY;
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                if (c0 < Dh) {
                    float v[32];
                    umma::tmem_ld32(tZ(q) + lo + (uint32_t)c0, v);
                    umma::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        zmax = fmaxf(zmax, v[j]);
                        zmin = fminf(zmin, v[j]);
                    }
                }
            }
            sp = 0.f;
            sn = 0.f;
            uint8_t *myQ = pq(q);
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                if (c0 < Dh) {
                    float v[32];
                    umma::tmem_ld32(tZ(q) + lo + (uint32_t)c0, v);
                    umma::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float a0 = __expf(v[j] - zmax), a1 = __expf(v[j + 1] - zmax);
                        const float b0 = __expf(zmin - v[j]), b1 = __expf(zmin - v[j + 1]);
                        sp += a0 + a1;
                        sn += b0 + b1;
                        pk[j >> 1] = umma::pack_bf16x2(a0, a1);
                        E1[(c0 + j) >> 1] = umma::pack_bf16x2(b0, b1);
                    }
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        *(uint4 *)(myQ + umma::kmajor_offset(r, c0 + 8 * w, 128)) =
                            u4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
                }
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) umma::mbar_arrive(&bphq[0]);
        }
        // pass 0 done: O and G carry e+ without its normaliser; bring them to s-/s+ scale
        // and hand the e- features to pass 1
        if (ok && (ok = waitw(&bpass[0], 0, err))) {
            umma::fence_after_sync();
            const float f = sn / sp;
            tmem_scale(tO(q) + lo, d + 16, f);
            for (int c = 0; c < nchi; ++c) tmem_scale(tG(q, c) + lo, KT, f);
            umma::tmem_wait_st();
            uint8_t *myQ = pq(q);
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                if (c0 < Dh) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int e0 = (c0 + 8 * w) >> 1;
                        *(uint4 *)(myQ + umma::kmajor_offset(r, c0 + 8 * w, 128)) =
                            u4(E1[e0], E1[e0 + 1], E1[e0 + 2], E1[e0 + 3]);
                    }
                }
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) umma::mbar_arrive(&bphq[1]);
        }
        const float rsn = 1.f / sn;
        int u = 0;
        float lsum = 0.f;   // sum of the row's rounded weights (band and softmax), at shift m
        if (ok && (ok = waitw(&bpass[1], 0, err))) {
            umma::fence_after_sync();
            tmem_scale(tO(q) + lo, d + 16, rsn);   // O = phi(Q) H1, column d = phi(Q).s1
            umma::tmem_wait_st();
            // band chunks: weight -G / s- where the leaving pair was folded but is still
            // inside the window of the row's query (the softmax attends it there)
            for (int c = 0; c < nchi && ok; ++c) {
                if (c > 0 && !(ok = waitw(&pfree[q], (uint32_t)((u - 1) & 1), err))) break;
                const long long j0 = jL0 + (long long)c * KT;
                const int i0 = (int)(j0 - (t0 - eta));
                const unsigned f0 = __ballot_sync(kFull, j0 + lane < jL1 && llf[i0 + lane] != 0);
                const unsigned f1 = __ballot_sync(kFull, j0 + 32 + lane < jL1 && llf[i0 + 32 + lane] != 0);
                const unsigned long long fm = (unsigned long long)f0 | ((unsigned long long)f1 << 32);
                // keys j0 + jj with jj > p - eta - j0 are inside the row's window
                const unsigned long long inwin = ~prefix_mask(p - eta - j0);
                const unsigned long long sub = row_ok ? (fm & inwin) : 0ull;
                float gv[64];
                {
                    float v0[32], v1[32];
                    umma::tmem_ld32(tG(q, c) + lo, v0);
                    umma::tmem_ld32(tG(q, c) + lo + 32u, v1);
                    umma::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        gv[j] = v0[j];
                        gv[32 + j] = v1[j];
                    }
                }
                if (c == 0) {
                    umma::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) umma::mbar_arrive(&bread[q]);   // the score buffer may take S(0)
                }
#pragma unroll
                for (int j0w = 0; j0w < 64; j0w += 8) {
                    float w[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) w[jj] = ((sub >> (j0w + jj)) & 1ull) ? -gv[j0w + jj] * rsn : 0.f;
                    const uint4 pw = u4(umma::pack_bf16x2(w[0], w[1]), umma::pack_bf16x2(w[2], w[3]),
                                        umma::pack_bf16x2(w[4], w[5]), umma::pack_bf16x2(w[6], w[7]));
                    lsum += sum_bf16x8(pw.x, pw.y, pw.z, pw.w);
                    *(uint4 *)(myP + umma::kmajor_offset(r, j0w, 128)) = pw;
                }
                umma::fence_async_smem();
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) umma::mbar_arrive(&pfull[q]);
                ++u;
            }
            if (ok && nchi == 0) {
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) umma::mbar_arrive(&bread[q]);
            }
        }

        // ---- softmax key tiles
        float m = 0.f;
        const float scale = rsqrtf((float)d);
        const float c1 = scale * 1.4426950408889634f;   // e^{x scale} = 2^{x c1}
        for (int i = 0; i < n && ok; ++i) {
            if (!(ok = waitw(&sfull[q], (uint32_t)(i & 1), err))) break;
            umma::fence_after_sync();
            float sv[KT];
            {
                float v0[32], v1[32];
                umma::tmem_ld32(tG(q, 0) + lo, v0);
                umma::tmem_ld32(tG(q, 0) + lo + 32u, v1);
                umma::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    sv[j] = v0[j];
                    sv[32 + j] = v1[j];
                }
            }
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) umma::mbar_arrive(&sfree[q]);
            if (!(ok = waitw(&mfull[i % kMS], (uint32_t)((i / kMS) & 1), err))) break;
            const TileMeta &M = meta[i % kMS];
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
            const bool all_live = __all_sync(kFull, live == ~0ull);
            float tmax;
            {
                float t[32];
                if (all_live) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) t[j] = fmaxf(sv[j], sv[j + 32]);
                } else {
                    const uint32_t lo32 = (uint32_t)live, hi32 = (uint32_t)(live >> 32);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        t[j] = fmaxf((lo32 >> j) & 1u ? sv[j] : -INFINITY, (hi32 >> j) & 1u ? sv[j + 32] : -INFINITY);
                }
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                    for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
                tmax = t[0] * scale;
            }
            // lazy rescaling: the shift only moves when the row's maximum exceeds it by
            // more than kLazy (weights stay below e^kLazy; numerator and denominator share m)
            const bool grow_m = tmax > m + kLazy;
            const bool any_grow = __any_sync(kFull, grow_m);
            const float mnew = grow_m ? tmax : m;
            const float mc = mnew * 1.4426950408889634f;
            uint32_t pk[32];
            const uint32_t lo32 = (uint32_t)live, hi32 = (uint32_t)(live >> 32);
#pragma unroll
            for (int j = 0; j < KT; j += 2) {
                float e0 = umma::ex2_approx(fmaf(sv[j], c1, -mc));
                float e1 = umma::ex2_approx(fmaf(sv[j + 1], c1, -mc));
                if (!all_live) {
                    const uint32_t wm = j < 32 ? lo32 : hi32;
                    const int jb = j & 31;
                    e0 = (wm >> jb) & 1u ? e0 : 0.f;
                    e1 = (wm >> (jb + 1)) & 1u ? e1 : 0.f;
                }
                pk[j >> 1] = umma::pack_bf16x2(e0, e1);
            }
            // the previous product on O and this tile's weight buffer is complete
            if (u > 0 && !(ok = waitw(&pfree[q], (uint32_t)((u - 1) & 1), err))) break;
            if (any_grow) {
                umma::fence_after_sync();
                tmem_scale(tO(q) + lo, d + 16, grow_m ? __expf(m - tmax) : 1.f);
                umma::tmem_wait_st();
            }
            if (grow_m) lsum *= __expf(m - tmax);
            m = mnew;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                lsum += sum_bf16x8(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
                *(uint4 *)(myP + umma::kmajor_offset(r, 8 * w, 128)) =
                    u4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                umma::mbar_arrive(&pfull[q]);
                umma::mbar_arrive(&mempty[i % kMS]);
            }
            ++u;
        }

        // ---- normalise and store
        if (ok && (ok = waitw(&bdone, 0, err))) {
            umma::fence_after_sync();
            float v[16];
            umma::tmem_ld16(tO(q) + lo + (uint32_t)d, v);
            umma::tmem_wait_ld();
            const float rden = 1.f / (v[0] + lsum + dm.eps * __expf(-m));
            bf16 *out = (bf16 *)a.out;
            const size_t orow = ((size_t)b * a.n_call + (size_t)(t0 - a.pos0) + (size_t)(grow / gq)) * dm.Hq +
                                (size_t)hk * gq + grow % gq;
            for (int c0 = 0; c0 < d; c0 += 16) {
                umma::tmem_ld16(tO(q) + lo + (uint32_t)c0, v);
                umma::tmem_wait_ld();
                if (row_ok) {
                    *(uint4 *)(out + orow * d + c0) =
                        u4(umma::pack_bf16x2(v[0] * rden, v[1] * rden), umma::pack_bf16x2(v[2] * rden, v[3] * rden),
                           umma::pack_bf16x2(v[4] * rden, v[5] * rden), umma::pack_bf16x2(v[6] * rden, v[7] * rden));
                    *(uint4 *)(out + orow * d + c0 + 8) =
                        u4(umma::pack_bf16x2(v[8] * rden, v[9] * rden), umma::pack_bf16x2(v[10] * rden, v[11] * rden),
                           umma::pack_bf16x2(v[12] * rden, v[13] * rden),
                           umma::pack_bf16x2(v[14] * rden, v[15] * rden));
                }
            }
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == kWarpM) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tm, 512);
    }
}

}  // namespace

bool attn_ws_supported(const Dims &dm)
{
    WGeo g;
    return make_wgeo(dm, &g);
}

size_t attn_ws_smem_bytes(const Dims &dm)
{
    WGeo g;
    return make_wgeo(dm, &g) ? g.total : 0;
}

bool make_attn_maps(const Dims &dm, const AttnArgs &a, const void *phiK, AttnMaps *maps)
{
    const unsigned long long rows = (unsigned long long)dm.B * a.n_call;
    const unsigned long long rk = (unsigned long long)dm.ns * (dm.lam + dm.R + dm.Nmax);
    return make_map_3d(&maps->q, a.q, dm.d, dm.Hq, rows, dm.g, 128 / dm.g) &&
           make_map_3d(&maps->k, a.kin, dm.d, dm.Hkv, rows, 1, KT) &&
           make_map_3d(&maps->v, a.vin, dm.d, dm.Hkv, rows, 1, KT) &&
           make_row_map(&maps->phik, phiK, rk, dm.D, KT);
}

void launch_attn_ws(const Dims &dm, const DevState &S, const PrefillScratch &P, const AttnArgs &a,
                    const AttnMaps &maps, cudaStream_t stream)
{
    WGeo g;
    if (!make_wgeo(dm, &g)) return;
    KVSrc<bf16> src{(const bf16 *)S.KS, (const bf16 *)S.VS, (const bf16 *)S.KR, (const bf16 *)S.VR,
                    (const bf16 *)a.kin, (const bf16 *)a.vin, dm.lam, dm.R, a.n_call, dm.Hkv, dm.d,
                    a.pos0};
    const int tpi = (dm.C * dm.g + 127) / 128;
    const int cpi = (tpi + g.nq - 1) / g.nq;
    dim3 grid(a.m * cpi, dm.ns);
    cudaFuncSetAttribute(attn_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.total);
    attn_ws_kernel<<<grid, kThreads, g.total, stream>>>(dm, S, P, a, src, g, maps);
}

}  // namespace lola
