// Tensor-core version of the sequential part of LoLA's update interval
// (gist.science technical summary, "Inferentiestrategie"; the Self-Recall Error
// of "Het Self-Recall Error (SRE) Mechanisme") for bfloat16 inputs. One CTA per
// (batch, kv-head) stream walks the stream's intervals in order.
//
// The fp32 state lives in TMEM for the whole call: feature f of block
// bk = f / 128 is TMEM lane f % 128, columns [bk*NBa, bk*NBa + d) hold H[f][:],
// column bk*NBa + d holds s[f]. A fold is a tcgen05 MMA chain that accumulates
// into it, H_blk += Phi_F^T V_F and s_blk += Phi_F^T 1, with the tokens' phi rows
// and value rows used as N-contiguous operands exactly as they are stored. After
// each fold a bf16 image of the state is written to shared memory: H as an
// N-contiguous [feature][value dim] operand and s as row 0 of a 16-row K-major
// operand. The SRE of 128 candidates at a time is then one MMA chain
// Phi_Q [H | s] into TMEM, and one thread per candidate finishes
// || num / (den + eps) - v ||^2 with the candidate's value row.
//
// Scoring tiles arrive by TMA: a tile of 128 cached candidates is one contiguous
// block of slot-ordered phi rows (the phi array's rows [0, lam) mirror the cache
// slots; the kernel rewrites a slot's row when a new pair takes it), loaded as
// one 128-row box per 64 features; a tile of leaving pairs is contiguous too when
// they all come from this call (prefill) or from one unwrapped run of the ring
// (decode); other tiles gather four rows per instruction (tile::gather4). The
// fold operands are gathered by 16-byte copies.
//
// The kept set is the nK smallest order-preserving keys (SRE bits inverted,
// token index), found by an 8-pass radix select. Every pair that is not kept --
// evicted cached pairs and leaving pairs alike -- folds right after the
// selection, in one pass, so the state becomes the state at the interval's end.
// Prefill mode stores its image as the interval's snapshot for the attention,
// which subtracts the linear terms of the folded leaving pairs that are still
// inside a query's window (the softmax attends them there).
#include "lola_internal.cuh"
#include "scoring.cuh"
#include "umma.cuh"

namespace lola {

namespace {

using bf16 = __nv_bfloat16;
constexpr int kThreads = 256;
constexpr int kFoldTok = 64;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per tensor-core completion wait
#ifndef LOLA_CHAIN_CTAS
#define LOLA_CHAIN_CTAS 64   // CTAs a prefill chain may spread over (the attention keeps the rest)
#endif

struct Geo {
    int D, d, NB, NBa, FP, nblk, lam, Lmax, QC, nbuf;
    uint32_t ncols;
    size_t off_Bs, off_ones, off_X, off_X1, off_B1, off_part, off_keys, off_keys1, off_rank, off_lst, off_slotTok,
        off_slotVrow, off_free, off_keep, off_flag, off_lf, off_hist, off_scal, total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shared memory: [H image, N-contiguous FP x d][s image, K-major 16 x FP][ones, K-major 16 x 64]
// [X: nbuf SRE phi tiles (K-major 128 x FP) | fold A blocks + value rows][partial sums][ints]
__host__ __device__ inline Geo make_geo_n(const Dims &dm, int nbuf)
{
    Geo g{};
    g.D = dm.D;
    g.d = dm.d;
    g.NB = dm.d + 16;
    g.NBa = (g.NB + 31) / 32 * 32;  // TMEM column stride of each accumulator
    g.FP = (dm.D + 127) / 128 * 128;
    g.nblk = g.FP / 128;
    g.lam = dm.lam;
    g.Lmax = dm.Lmax;
    g.QC = dm.lam + dm.Lmax;
    g.nbuf = nbuf;
    const uint32_t need = (uint32_t)((g.nblk + 1) * g.NBa);
    g.ncols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
    size_t o = (size_t)g.FP * g.d * 2;                        // H image
    g.off_Bs = o;                                              // s image
    o += (size_t)g.FP * 32;
    g.off_ones = al(o, 1024);
    o = g.off_ones + 16 * 64 * 2;
    g.off_X = al(o, 1024);
    const size_t tile = (size_t)128 * g.FP * 2;
    g.off_X1 = g.off_X + tile;
    const size_t xs = (size_t)nbuf * tile;
    const size_t xf = (size_t)g.nblk * 64 * 128 * 2 + (size_t)64 * g.d * 2;
    g.off_B1 = g.off_X + (size_t)g.nblk * 64 * 128 * 2;
    o = g.off_X + (xs > xf ? xs : xf);
    g.off_part = al(o, 16);
    o = g.off_part + 128 * 4;
    g.off_keys = al(o, 16);
    o = g.off_keys + (size_t)g.QC * 4;
    g.off_keys1 = o;                                           // second key buffer (odd intervals)
    o += (size_t)g.QC * 4;
    g.off_rank = o;
    o += (size_t)g.QC * 4;
    g.off_lst = o;
    o += (size_t)g.QC * 4;
    g.off_slotTok = o;
    o += (size_t)g.lam * 4;
    g.off_slotVrow = o;
    o += (size_t)g.lam * 4;
    g.off_free = o;
    o += (size_t)g.lam * 2;
    g.off_keep = o;
    o += (size_t)g.QC;
    g.off_flag = o;
    o += (size_t)g.QC;
    g.off_lf = o;
    o += (size_t)g.Lmax;
    g.off_hist = al(o, 16);
    o = g.off_hist + 2 * 256 * 4;
    g.off_scal = o;
    o += 64 * 4;
    g.total = o + 1024;  // alignment slack for the 1024-byte aligned base
    if (g.ncols == 512 && g.total < 116 * 1024) g.total = 116 * 1024;  // one CTA per SM
    return g;
}

// Two SRE tile buffers (the next tile loads while this one is scored) when they fit.
__host__ __device__ inline Geo make_geo(const Dims &dm)
{
    const Geo g2 = make_geo_n(dm, 2);
    return g2.total <= 227 * 1024 - 64 ? g2 : make_geo_n(dm, 1);
}

template <typename F>
__device__ int scan_excl(const F *in, int *out, int n, int *wsum)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int beg = min(n, tid * per), end = min(n, beg + per);
    int local = 0;
    for (int i = beg; i < end; ++i) local += (int)in[i];
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
        run += (int)in[i];
    }
    const int total = wsum[nwarps - 1];
    __syncthreads();
    return total;
}

// The k-th smallest (1-based) of n distinct 64-bit keys key(c) = (hi[c] << 32) | tok(c),
// 8 bits per pass; the two histograms alternate so each pass needs two barriers.
template <typename TokF>
__device__ unsigned long long radix_select(const unsigned *hi, TokF tok, int n, int k, int *hist2,
                                           int *scal)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long prefix = 0, mask = 0;
    int rank = k;
    for (int i = tid; i < 256; i += nt) hist2[i] = 0;
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        int *hist = hist2 + (pass & 1) * 256;
        int *other = hist2 + ((pass + 1) & 1) * 256;
        for (int c = tid; c < n; c += nt) {
            const unsigned long long kk = ((unsigned long long)hi[c] << 32) | (unsigned)tok(c);
            if ((kk & mask) == prefix) atomicAdd(&hist[(int)((kk >> shift) & 255u)], 1);
        }
        for (int i = tid; i < 256; i += nt) other[i] = 0;
        __syncthreads();
        if (warp == 0) {
            int loc[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                loc[j] = hist[lane * 8 + j];
                s += loc[j];
            }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - s;
            if (excl < rank && rank <= incl) {
                int cum = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum + loc[j] >= rank) {
                        scal[0] = lane * 8 + j;
                        scal[1] = rank - cum;
                        scal[4] = loc[j];          // keys sharing the extended prefix
                        break;
                    }
                    cum += loc[j];
                }
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)scal[0] << shift;
        mask |= (unsigned long long)255u << shift;
        rank = scal[1];
        if (scal[4] == 1) {
            // a single key carries this prefix: it is the answer
            __syncthreads();
            for (int c = tid; c < n; c += nt) {
                const unsigned long long kk = ((unsigned long long)hi[c] << 32) | (unsigned)tok(c);
                if ((kk & mask) == prefix) *(unsigned long long *)(scal + 6) = kk;
            }
            __syncthreads();
            const unsigned long long r = *(const unsigned long long *)(scal + 6);
            __syncthreads();
            return r;
        }
    }
    __syncthreads();
    return prefix;
}

struct Ctx {
    Geo g;
    uint8_t *Bimg;          // H image (N-contiguous [FP][d]), followed by the s image
    uint8_t *Bs, *ones, *X;
    uint32_t tm;           // TMEM base
    uint64_t *mbar;
    const CUtensorMap *phimap;   // phi rows of this launch, [ns * nvrows][D]
    long long row0;        // map row of this stream's virtual row 0
    int oob_row;           // a map row past the extent (reads as zeros)
    int *okflag;
    int *err;              // device error word (timeouts stop every CTA's waits)
    uint32_t phase;
};

__device__ __forceinline__ uint32_t tH(const Ctx &c, int bk) { return c.tm + (uint32_t)(bk * c.g.NBa); }
__device__ __forceinline__ uint32_t tS(const Ctx &c) { return c.tm + (uint32_t)(c.g.nblk * c.g.NBa); }

__device__ bool wait_mma(Ctx &c)
{
    if (threadIdx.x == 0) {
        const bool ok = umma::mbar_wait_abortable(c.mbar, c.phase, kWaitNs, c.err, ERR_TIMEOUT);
        if (!ok) raise_error(c.err, ERR_TIMEOUT);
        *c.okflag = ok ? 1 : 0;
    }
    __syncthreads();
    c.phase ^= 1u;
    umma::fence_after_sync();
    return *c.okflag != 0;
}

// bf16 images of the state: H as an N-contiguous [feature][value dim] operand
// (16-byte stores of 8 value dims), s as row 0 of a K-major 16 x FP operand.
__device__ void refresh_image(Ctx &c)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = warp & 3;
    // the last snapshot store must have read the image before it is overwritten
    if (threadIdx.x == 0) umma::bulk_wait_read();
    __syncthreads();
    // units of (feature block, 16-column piece or the s column), dealt to the two
    // groups of four warps; warp w reads TMEM lanes 32 * (w % 4) ..
    const int npc = c.g.d / 16 + 1;
    for (int u = warp >> 2; u < c.g.nblk * npc; u += kThreads / 128) {
        const int bk = u / npc, cc = u - bk * npc;
        const int f = bk * 128 + q * 32 + lane;
        const uint32_t row = tH(c, bk) + ((uint32_t)(q * 32) << 16);
        float v[16];
        if (cc * 16 < c.g.d) {
            const int c0 = cc * 16;
            umma::tmem_ld16(row + (uint32_t)c0, v);
            umma::tmem_wait_ld();
            uint4 h0, h1;
            h0.x = umma::pack_bf16x2(v[0], v[1]);
            h0.y = umma::pack_bf16x2(v[2], v[3]);
            h0.z = umma::pack_bf16x2(v[4], v[5]);
            h0.w = umma::pack_bf16x2(v[6], v[7]);
            h1.x = umma::pack_bf16x2(v[8], v[9]);
            h1.y = umma::pack_bf16x2(v[10], v[11]);
            h1.z = umma::pack_bf16x2(v[12], v[13]);
            h1.w = umma::pack_bf16x2(v[14], v[15]);
            *(uint4 *)(c.Bimg + umma::mnmajor_offset(f, c0, c.g.d)) = h0;
            *(uint4 *)(c.Bimg + umma::mnmajor_offset(f, c0 + 8, c.g.d)) = h1;
        } else {
            umma::tmem_ld16(row + (uint32_t)c.g.d, v);
            umma::tmem_wait_ld();
            *(bf16 *)(c.Bs + umma::kmajor_offset(0, f, 16)) = __float2bfloat16_rn(v[0]);
        }
    }
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
}

// H += sum phi(k) v^T, s += sum phi(k) over the listed virtual rows, on the tensor
// cores. A = the tokens' phi rows and B = their value rows, both N-contiguous
// as stored (copied with 16-byte cp.async, no transpose); a second MMA against
// a ones column accumulates s in column d.
__device__ bool fold_tc(Ctx &c, const int *lst, int cnt, const bf16 *__restrict__ phi_st,
                        const KVSrc<bf16> &src, int st)
{
    const int tid = threadIdx.x;
    const Geo &g = c.g;
    uint8_t *Af = c.X;                                              // nblk x [64 tokens x 128 features]
    uint8_t *B1 = c.X + (size_t)g.nblk * 64 * 128 * 2;              // [64 tokens x d]
    const uint32_t id_h = umma::idesc_bf16(128, g.d, true, true);
    const uint32_t id_s = umma::idesc_bf16(128, 16, true, false);
    const int lgf = __ffs(g.FP >> 3) - 1, lgv = __ffs(g.d >> 3) - 1;  // 16-byte chunks per row
    for (int base = 0; base < cnt; base += kFoldTok) {
        const int nt = min(kFoldTok, cnt - base);
        const int ntp = (nt + 15) & ~15;
        // A = Phi_F^T, MN-major per 128-feature block (16-byte copies; tokens past nt
        // and features past D are zeros)
        for (int e = tid; e < (ntp << lgf); e += kThreads) {
            const int t = e >> lgf, f = (e & ((1 << lgf) - 1)) * 8;
            uint8_t *dst = Af + (size_t)(f >> 7) * 64 * 128 * 2 + umma::mnmajor_offset(t, f & 127, 128);
            if (t < nt && f < g.D) umma::cp_async16(dst, phi_st + (size_t)lst[base + t] * g.D + f);
            else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
        for (int e = tid; e < (ntp << lgv); e += kThreads) {
            const int t = e >> lgv, c0 = (e & ((1 << lgv) - 1)) * 8;
            uint8_t *dst = B1 + umma::mnmajor_offset(t, c0, g.d);
            if (t < nt) umma::cp_async16(dst, src.vrow(st, lst[base + t]) + c0);
            else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
        umma::cp_async_commit();
        umma::cp_async_wait_all();
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0 || tid == 32) {
            // two issuing threads, value columns (thread 0) and the normaliser column
            // (thread 32): different TMEM columns, issued side by side; both commit
            umma::fence_after_sync();
            const uint32_t b1 = umma::smem_u32(B1), on = umma::smem_u32(c.ones);
            for (int bk = 0; bk < g.nblk; ++bk) {
                const uint32_t a0 = umma::smem_u32(Af + (size_t)bk * 64 * 128 * 2);
                for (int ks = 0; ks < ntp / 16; ++ks) {
                    const uint64_t ad = umma::mnmajor_desc(a0, ks, 128);
                    if (tid == 0) umma::mma_ss(tH(c, bk), ad, umma::mnmajor_desc(b1, ks, g.d), id_h, 1u);
                    else umma::mma_ss(tH(c, bk) + (uint32_t)g.d, ad, umma::kmajor_desc(on, ks, 16), id_s, 1u);
                }
            }
            umma::mma_commit(c.mbar);
        }
        if (!wait_mma(c)) return false;
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    chain_tc_kernel(Dims dm, DevState S, PrefillScratch P, ChainArgs a, KVSrc<bf16> src, int nc,
                    const __grid_constant__ CUtensorMap phimap, const __grid_constant__ CUtensorMap boxmap)
{
    // nc > 1: a cluster of nc CTAs per stream; every CTA holds the state and applies the
    // same folds, the SRE tiles are dealt round-robin, the keys are exchanged through
    // distributed shared memory, and rank 0 alone writes to global memory
    const int st = blockIdx.x / nc;
    const int crank = nc > 1 ? (int)umma::cluster_ctarank() : 0;
    const bool lead = crank == 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const Geo g = make_geo(dm);
    const int D = g.D, d = g.d, lam = g.lam, eta = dm.eta, Lmax = g.Lmax;

    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar;
    __shared__ uint64_t tbar[2];     // SRE tile buffer 0 / 1 has landed
    __shared__ uint64_t never;       // nothing arrives here (fault-injection hook)
    __shared__ uint64_t kready[2];   // peers' keys of an even / odd interval have arrived
    __shared__ uint32_t tslot;
    __shared__ int okflag;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    Ctx c;
    c.g = g;
    c.Bimg = base;
    c.Bs = base + g.off_Bs;
    c.ones = base + g.off_ones;
    c.X = base + g.off_X;
    unsigned *keys0 = (unsigned *)(base + g.off_keys);     // high 32 bits of each candidate's key
    unsigned *keys1 = (unsigned *)(base + g.off_keys1);    // (two buffers: even / odd intervals)
    int *rank = (int *)(base + g.off_rank);
    int *lst = (int *)(base + g.off_lst);
    int *slotTok = (int *)(base + g.off_slotTok);
    int *slotVrow = (int *)(base + g.off_slotVrow);
    short *freeSlot = (short *)(base + g.off_free);
    uint8_t *keep = base + g.off_keep;
    uint8_t *flag = base + g.off_flag;
    uint8_t *lf = base + g.off_lf;
    int *hist = (int *)(base + g.off_hist);
    int *scal = (int *)(base + g.off_scal);
    c.mbar = &mbar;
    c.phimap = &phimap;
    c.row0 = (long long)st * a.nvrows;
    c.oob_row = dm.ns * a.nvrows;
    c.okflag = &okflag;
    c.err = S.err;
    c.phase = 0;
    // thread 0 (lane 0 of the issuing warp): tile loads issued into / waited for per buffer
    uint32_t tiss[2] = {0u, 0u}, twait[2] = {0u, 0u};
    // constant operands: s image rows 1..15 and the ones column (row 0 of a 16 x 64 tile)
    for (int e = tid; e < g.FP * 16; e += kThreads) {
        const int r = e / g.FP, f = e - r * g.FP;
        if (r > 0) *(bf16 *)(c.Bs + umma::kmajor_offset(r, f, 16)) = __float2bfloat16_rn(0.f);
    }
    for (int e = tid; e < 16 * 64; e += kThreads) {
        const int r = e / 64, k = e - r * 64;
        *(bf16 *)(c.ones + umma::kmajor_offset(r, k, 16)) = __float2bfloat16_rn(r == 0 ? 1.f : 0.f);
    }

    if (tid == 0) {
        umma::mbar_init(&mbar, 2);   // two issuing threads commit per MMA batch
        umma::mbar_init(&tbar[0], 1);
        umma::mbar_init(&tbar[1], 1);
        umma::mbar_init(&never, 1);
        umma::mbar_init(&kready[0], nc > 1 ? nc - 1 : 1);
        umma::mbar_init(&kready[1], nc > 1 ? nc - 1 : 1);
    }
    if (warp == 0) umma::tmem_alloc(&tslot, g.ncols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    if (nc > 1) umma::cluster_sync();   // every peer's barriers exist before anyone arrives
    c.tm = tslot;

    float *Hg = S.H + (size_t)st * D * d;
    float *sg = S.s + (size_t)st * D;
    const bf16 *phi_st = (const bf16 *)a.phi + (size_t)st * a.nvrows * D;

    // state -> TMEM (rows past D and columns past d+1 are zero)
    {
        const int q = warp & 3;
        for (int bk = warp >> 2; bk < g.nblk; bk += kThreads / 128) {
            const int f = bk * 128 + q * 32 + lane;
            for (int c0 = 0; c0 < g.NB; c0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int col = c0 + i;
                    v[i] = f < D ? (col < d ? Hg[(size_t)f * d + col] : (col == d ? sg[f] : 0.f)) : 0.f;
                }
                umma::tmem_st16(tH(c, bk) + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
            }
        }
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
    }
    refresh_image(c);

    int nS = a.nS0;
    for (int i = tid; i < lam; i += kThreads) {
        if (a.mode == 0 && a.cont) {
            slotTok[i] = P.slotTok[(size_t)st * lam + i];
            // written by the previous launch of this call; clamped so that a launch after
            // one that gave up (error word set, scratch not written) stays in bounds
            slotVrow[i] = min(max(P.slotVrow[(size_t)st * lam + i], 0), a.nvrows - 1);
        } else {
            slotTok[i] = i < nS ? S.idxS[(size_t)st * lam + i] : -1;
            slotVrow[i] = i;
        }
    }
    for (int i = tid; i < Lmax; i += kThreads) lf[i] = i < a.pend_n ? S.pend[(size_t)st * Lmax + i] : 0;
    int pend_n = a.pend_n;
    __syncthreads();

    bool ok = true;
    int seg_sig = 0;   // segments of the call counted in a.seg_done (lead CTA, thread 0)
    const uint32_t id_sh = umma::idesc_bf16(128, d, false, true);
    const uint32_t id_ss = umma::idesc_bf16(128, 16, false, false);
    for (int ci = 0; ci < a.n_int && ok; ++ci) {
        const long long t0 = a.pos0 + (long long)ci * a.ilen;
        const long long t1 = t0 + a.ilen;
        const long long iglob = a.iglob0 + ci;

        if (a.inject_ns != 0 && ci == 0) {
            // test hook: a bounded wait that runs out, handled like any other timeout
            if (tid == 0) {
                const bool got = umma::mbar_wait(&never, 0, a.inject_ns);
                if (!got) raise_error(S.err, ERR_TIMEOUT);
                okflag = got ? 1 : 0;
            }
            __syncthreads();
            if (!(ok = okflag != 0)) break;
        }
        unsigned *keys = (ci & 1) ? keys1 : keys0;
        // 2. score the candidates (cache slots, then pairs leaving in [t0, t1))
        const long long Llo = t0 - eta > 0 ? t0 - eta : 0;
        const long long Lhi = t1 - eta > Llo ? t1 - eta : Llo;
        const int nL = (int)(Lhi - Llo);
        const int nQ = nS + nL;
        // virtual row of every candidate, once per interval (rank[] is free here)
        int *cvrow = rank;
        for (int cnd = tid; cnd < nQ; cnd += kThreads)
            cvrow[cnd] = cnd < nS ? slotVrow[cnd] : src.tok2vrow(Llo + (cnd - nS));
        __syncthreads();
        if (dm.scorer != kScoreSRE) {
            // an ablation score instead of the SRE: every CTA scores every candidate (no
            // key exchange); the first-query rows come from the caller's queries
            float *score = (float *)keys;
            float *lg = (float *)lst, *lu = (float *)((ci & 1) ? keys0 : keys1);
            float *qs = (float *)c.X, *pq = qs + dm.g * d, *red = (float *)(base + g.off_part);
            const bf16 *qb = (const bf16 *)a.qin;
            const int b = st / dm.Hkv, hk = st % dm.Hkv;
            const size_t qrow0 = (((size_t)b * a.q_n + (size_t)(t0 - a.q_start)) * dm.Hq + (size_t)hk * dm.g) * d;
            alt_scores<bf16>(
                dm.scorer, nQ, [&](int cc) { return src.krow(st, cvrow[cc]); },
                [&](int cc) { return phi_st + (size_t)cvrow[cc] * D; },
                [&](int h) { return qb + qrow0 + (size_t)h * d; },
                [&](int cc) { return cc < nS ? slotTok[cc] : (int)(Llo + (cc - nS)); }, w_of(dm, S.W, hk), dm.g, d, D, score,
                qs, pq, lg, lu, red);
            for (int cc = tid; cc < nQ; cc += kThreads) {
                const float sc = score[cc];
                if (a.score_sre != nullptr && iglob < a.score_cap && lead) {
                    const size_t o = ((size_t)iglob * dm.ns + st) * g.QC + cc;
                    a.score_sre[o] = sc;
                    a.score_tok[o] = cc < nS ? slotTok[cc] : (int)(Llo + (cc - nS));
                }
                keys[cc] = 0xFFFFFFFFu - __float_as_uint(fmaxf(sc, 0.f));
            }
            __syncthreads();
        }
        const int ntile = dm.scorer == kScoreSRE ? (nQ + 127) / 128 : 0;
        const int nmy = ntile > crank ? (ntile - crank + nc - 1) / nc : 0;   // this CTA's tiles
        // phi rows of this CTA's tile lt (K-major A operand) into buffer lt % nbuf by TMA
        // row gathers from warp 0 (rows r..r+3 of one 64-feature block per instruction;
        // rows past the candidates read as zeros); completion on tbar[buffer]
        auto load_tile = [&](int lt) {
            if (warp != 0) return;
            const int bsel = lt % g.nbuf;
            uint8_t *dstT = base + (bsel ? g.off_X1 : g.off_X);
            const int m0 = (crank + lt * nc) * 128, nr = min(128, nQ - m0);
            const int natom = g.FP >> 6;
            if (lane == 0) {
                umma::mbar_arrive_expect_tx(&tbar[bsel], (uint32_t)(128 * g.FP * 2));
                ++tiss[bsel];
            }
            __syncwarp();
            // one contiguous run of phi rows: 128-row boxes (rows past the tile's
            // candidates are other rows of the array or zeros; their scores are unused)
            long long brow = -1;
            if (m0 + 128 <= nS) {
                brow = m0;                                  // cached candidates = slots m0..
            } else if (m0 >= nS) {
                const long long t0L = Llo + (m0 - nS);      // first leaving pair of the tile
                if (a.mode == 0 ? t0L >= a.call_start
                                : ((int)(t0L & (dm.R - 1)) + nr <= dm.R))
                    brow = src.tok2vrow(t0L);
            }
            if (brow >= 0) {
                if (lane < natom)
                    umma::tma_load_2d(dstT + umma::kmajor_row(0, lane, 128), &boxmap, lane * 64,
                                      (int)(c.row0 + brow), &tbar[bsel]);
                return;
            }
            for (int e = lane; e < 32 * natom; e += 32) {
                const int grp = e / natom, at = e - grp * natom;
                const int r = grp * 4;
                int rr[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) rr[i] = r + i < nr ? (int)(c.row0 + cvrow[m0 + r + i]) : c.oob_row;
                umma::gather4(dstT + umma::kmajor_row(r, at, 128), c.phimap, at * 64, rr[0], rr[1], rr[2], rr[3],
                              &tbar[bsel]);
            }
        };
        if (nmy > 0) load_tile(0);
        if (g.nbuf == 2 && nmy > 1) load_tile(1);
        const int q = warp & 3, half = warp >> 2;
        const int r = q * 32 + lane;                      // this thread's row of the tile
        const int hd = d >> 1;                            // value dims per thread
        for (int lt = 0; lt < nmy && ok; ++lt) {
            const int m0 = (crank + lt * nc) * 128, nr = min(128, nQ - m0);
            if (tid == 0 || tid == 32) {
                // the tile's rows have landed (a timeout stops the MMA wait below at once);
                // thread 0 issues the numerator columns, thread 32 the denominator column
                const int bsel = lt % g.nbuf;
                const bool got = umma::mbar_wait_abortable(&tbar[bsel], twait[bsel] & 1u, kWaitNs, S.err, ERR_TIMEOUT);
                if (got) ++twait[bsel];
                else raise_error(S.err, ERR_TIMEOUT);   // the MMA wait below gives up at once
                umma::fence_after_sync();
                const uint32_t a0 = umma::smem_u32(base + (bsel ? g.off_X1 : g.off_X));
                const uint32_t bh = umma::smem_u32(c.Bimg), bs = umma::smem_u32(c.Bs);
                for (int ks = 0; ks < g.FP / 16; ++ks) {
                    const uint64_t ad = umma::kmajor_desc(a0, ks, 128);
                    if (tid == 0) umma::mma_ss(tS(c), ad, umma::mnmajor_desc(bh, ks, d), id_sh, ks > 0 ? 1u : 0u);
                    else umma::mma_ss(tS(c) + (uint32_t)d, ad, umma::kmajor_desc(bs, ks, 16), id_ss, ks > 0 ? 1u : 0u);
                }
                umma::mma_commit(c.mbar);
            }
            // this thread's half of its candidate's value row, fetched while the MMA runs
            uint4 vr4[8];
            if (r < nr) {
                const uint4 *vsrc = (const uint4 *)(src.vrow(st, cvrow[m0 + r]) + half * hd);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i * 8 < hd) vr4[i] = vsrc[i];
            }
            if (!(ok = wait_mma(c))) break;
            if (g.nbuf == 1 && lt + 1 < nmy) load_tile(lt + 1);         // the tile buffer is free
            if (g.nbuf == 2 && lt + 2 < nmy) load_tile(lt + 2);
            {
                const uint32_t rowaddr = tS(c) + ((uint32_t)(q * 32) << 16);
                float v[16];
                umma::tmem_ld16(rowaddr + (uint32_t)d, v);
                umma::tmem_wait_ld();
                const float den = v[0] + dm.eps;
                const float rden = den != 0.f ? 1.f / den : 0.f;
                float err = 0.f;
#pragma unroll
                for (int i2 = 0; i2 < 4; ++i2) {
                    if (i2 * 16 < hd) {
                        umma::tmem_ld16(rowaddr + (uint32_t)(half * hd + i2 * 16), v);
                        umma::tmem_wait_ld();
                        const bf16 *p0 = (const bf16 *)&vr4[2 * i2];
                        const bf16 *p1 = (const bf16 *)&vr4[2 * i2 + 1];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float diff = v[i] * rden - __bfloat162float(i < 8 ? p0[i] : p1[i - 8]);
                            err = fmaf(diff, diff, err);
                        }
                    }
                }
                float *part = (float *)(base + g.off_part);
                if (half == 1) part[r] = err;
                __syncthreads();
                if (half == 0 && r < nr) {
                    err += part[r];
                    keys[m0 + r] = 0xFFFFFFFFu - __float_as_uint(fmaxf(err, 0.f));
                    if (a.score_sre != nullptr && iglob < a.score_cap) {
                        const int cand = m0 + r;
                        const size_t o = ((size_t)iglob * dm.ns + st) * g.QC + cand;
                        a.score_sre[o] = err;
                        a.score_tok[o] = cand < nS ? slotTok[cand] : (int)(Llo + (cand - nS));
                    }
                }
            }
            umma::fence_before_sync();
            __syncthreads();
        }
        if (!ok) break;
        if (nc > 1 && dm.scorer == kScoreSRE) {
            // push this CTA's keys into every peer's buffer, then signal it; wait for theirs
            for (int pr = 1; pr < nc; ++pr) {
                const uint32_t peer = (uint32_t)((crank + pr) % nc);
                const uint32_t rk = umma::cluster_map(keys, peer);
                for (int lt = 0; lt < nmy; ++lt) {
                    const int m0 = (crank + lt * nc) * 128, nr = min(128, nQ - m0);
                    for (int i = tid; i < nr; i += kThreads)
                        umma::st_cluster_u32(rk + (uint32_t)(m0 + i) * 4u, keys[m0 + i]);
                }
            }
            __syncthreads();
            if (tid == 0) {
                umma::fence_cluster();
                for (int pr = 1; pr < nc; ++pr)
                    umma::mbar_arrive_cluster(umma::cluster_map(&kready[ci & 1], (uint32_t)((crank + pr) % nc)));
                const bool got = umma::mbar_wait_cluster_abortable(&kready[ci & 1], (uint32_t)((ci >> 1) & 1), kWaitNs,
                                                                   S.err, ERR_TIMEOUT);
                if (!got) raise_error(S.err, ERR_TIMEOUT);
                okflag = got ? 1 : 0;
            }
            __syncthreads();
            if (!(ok = okflag != 0)) break;
        }

        // 3. keep the nK smallest keys (highest SRE, lower token on ties)
        const int nK = nQ < lam ? nQ : lam;
        auto tok_of = [&](int i) -> int { return i < nS ? slotTok[i] : (int)(Llo + (i - nS)); };
        if (nQ > lam) {
            const unsigned long long thr = radix_select(keys, tok_of, nQ, nK, hist, scal);
            for (int i = tid; i < nQ; i += kThreads) {
                const unsigned long long kk = ((unsigned long long)keys[i] << 32) | (unsigned)tok_of(i);
                keep[i] = kk <= thr ? 1 : 0;
            }
        } else {
            for (int i = tid; i < nQ; i += kThreads) keep[i] = 1;
        }
        __syncthreads();
        if (a.sel_log != nullptr && iglob < a.sel_cap && lead) {
            int32_t *lg = a.sel_log + ((size_t)iglob * dm.ns + st) * (lam + 1);
            const int cnt = scan_excl(keep, rank, nQ, scal);
            for (int i = tid; i < nQ; i += kThreads)
                if (keep[i]) lg[1 + rank[i]] = i < nS ? slotTok[i] : (int)(Llo + (i - nS));
            for (int i = cnt + tid; i < lam; i += kThreads) lg[1 + i] = -1;
            if (tid == 0) lg[0] = cnt;
        }
        const int32_t *lo_ =
            (a.ovr != nullptr && iglob < a.ovr_n) ? a.ovr + ((size_t)iglob * dm.ns + st) * (lam + 1) : nullptr;
        if (lo_ != nullptr && lo_[0] >= 0) {
            const int cnt = lo_[0];
            if (tid == 0 && cnt != nK) raise_error(S.err, ERR_BOUNDS);
            for (int i = tid; i < nQ; i += kThreads) {
                const int key = i < nS ? slotTok[i] : (int)(Llo + (i - nS));
                int lo = 0, hi = cnt < lam ? cnt : lam;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (lo_[1 + mid] < key) lo = mid + 1; else hi = mid;
                }
                keep[i] = (lo < cnt && lo < lam && lo_[1 + lo] == key) ? 1 : 0;
            }
            __syncthreads();
        }

        // 4a. every pair that is not kept -- evicted cached pairs and leaving pairs --
        //     folds now, in one pass: the state becomes the state at the interval's end
        for (int i = tid; i < nQ; i += kThreads) flag[i] = keep[i] ? 0 : 1;
        __syncthreads();
        const int nE = scan_excl(flag, rank, nS, scal);
        for (int i = tid; i < nS; i += kThreads) {
            if (flag[i]) {
                lst[rank[i]] = slotVrow[i];
                freeSlot[rank[i]] = (short)i;
            }
        }
        for (int r = nE + tid; r < nE + (lam - nS); r += kThreads) freeSlot[r] = (short)(nS + (r - nE));
        __syncthreads();
        const int nLf = scan_excl(flag + nS, rank, nL, scal);
        for (int i = tid; i < nL; i += kThreads)
            if (flag[nS + i]) lst[nE + rank[i]] = src.tok2vrow(Llo + i);
        __syncthreads();
        if (nE + nLf > 0) {
            if (!(ok = fold_tc(c, lst, nE + nLf, phi_st, src, st))) break;
            refresh_image(c);
        }
        if (a.mode == 0 && P.snapImg != nullptr && tid == 0 && lead) {
            // the image (written and proxy-fenced by refresh_image) goes out as one bulk store
            uint8_t *dst = (uint8_t *)P.snapImg + ((size_t)st * dm.mmax + a.ci0 + ci) * g.NB * g.FP * 2;
            umma::bulk_s2g(dst, c.Bimg, (uint32_t)(g.NB * g.FP * 2));
        }
        if (a.mode == 0 && a.snap_f32 && lead) {
            // fp32 (H', s') for the SIMT attention kernel
            const int q = warp & 3;
            float *sh = P.snapH + ((size_t)st * dm.mmax + a.ci0 + ci) * D * d;
            float *ss = P.snapS + ((size_t)st * dm.mmax + a.ci0 + ci) * D;
            for (int bk = warp >> 2; bk < g.nblk; bk += kThreads / 128) {
                const int f = bk * 128 + q * 32 + lane;
                for (int c0 = 0; c0 < g.NB; c0 += 16) {
                    float v[16];
                    umma::tmem_ld16(tH(c, bk) + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
                    umma::tmem_wait_ld();
                    if (f < D) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int col = c0 + i;
                            if (col < d) sh[(size_t)f * d + col] = v[i];
                            else if (col == d) ss[f] = v[i];
                        }
                    }
                }
            }
        }

        // 4b. kept leaving pairs take the free slots (eviction slots first, ascending)
        const int nNew = scan_excl(keep + nS, rank, nL, scal);
        if (tid == 0 && nNew > nE + (lam - nS)) raise_error(S.err, ERR_BOUNDS);
        for (int i = tid; i < nL; i += kThreads) {
            if (keep[nS + i] && rank[i] < nE + (lam - nS)) {
                const int slot = freeSlot[rank[i]];
                const long long tok = Llo + i;
                slotTok[slot] = (int)tok;
                slotVrow[slot] = a.mode == 0 ? src.tok2vrow(tok) : slot;
            }
        }
        if (a.mode == 0) {
            // the slot's phi row follows its new pair (only the CTA that scores the
            // slot's tile reads that row back, by TMA: fence for the async proxy)
            bf16 *phw = (bf16 *)a.phi + (size_t)st * a.nvrows * D;
            bool wrote = false;
            for (int i = warp; i < nL; i += kThreads / 32) {
                if (!keep[nS + i] || rank[i] >= nE + (lam - nS)) continue;
                const int slot = freeSlot[rank[i]];
                if ((slot >> 7) % nc != crank) continue;
                const uint4 *from = (const uint4 *)(phw + (size_t)src.tok2vrow(Llo + i) * D);
                uint4 *to = (uint4 *)(phw + (size_t)slot * D);
                for (int e = lane; e < D / 8; e += 32) to[e] = from[e];
                wrote = true;
            }
            if (wrote) umma::fence_async_global();
        }
        if (a.mode == 1) {
            bf16 *KS = (bf16 *)S.KS + (size_t)st * lam * d;
            bf16 *VS = (bf16 *)S.VS + (size_t)st * lam * d;
            bf16 *phiV = (bf16 *)S.phiV + (size_t)st * a.nvrows * D;
            for (int i = warp; i < nL; i += kThreads / 32) {
                if (!keep[nS + i] || rank[i] >= nE + (lam - nS)) continue;
                const int slot = freeSlot[rank[i]];
                const int vr = src.tok2vrow(Llo + i);
                const bf16 *kr = src.krow(st, vr);
                const bf16 *vv = src.vrow(st, vr);
                for (int e = lane; e < d; e += 32) {
                    KS[(size_t)slot * d + e] = kr[e];
                    VS[(size_t)slot * d + e] = vv[e];
                }
                for (int e = lane; e < D; e += 32) phiV[(size_t)slot * D + e] = phiV[(size_t)vr * D + e];
                if (lane == 0) S.idxS[(size_t)st * lam + slot] = (int)(Llo + i);
            }
        }
        __syncthreads();
        if (a.mode == 0 && lead) {
            const size_t lb = (size_t)st * dm.mmax + a.ci0 + ci;
            for (int i = tid; i < nK; i += kThreads) {
                P.logTok[lb * lam + i] = slotTok[i];
                P.logVrow[lb * lam + i] = slotVrow[i];
            }
            for (int i = tid; i < nL; i += kThreads)
                P.logLf[lb * Lmax + (int)(Llo + i - (t0 - eta))] = keep[nS + i] ? 0 : 1;
            if (tid == 0) P.logCount[lb] = nK;
        }
        __syncthreads();
        for (int i = tid; i < nL; i += kThreads) lf[i] = keep[nS + i] ? 0 : 1;
        pend_n = nL;
        nS = nK;
        __syncthreads();
        if (a.seg_done != nullptr && lead && tid == 0 && ((ci + 1) % a.seg_len == 0 || ci == a.n_int - 1)) {
            // this stream's intervals of the segment are done: its logs (plain stores) and
            // snapshot images (bulk stores, waited for here) are visible before the count
            umma::bulk_wait_all();
            umma::fence_async_global();
            __threadfence();
            atomicAdd(&a.seg_done[ci / a.seg_len], 1);
            seg_sig = ci / a.seg_len + 1;
        }
    }

    if (ok && lead) {
        // TMEM -> state
        const int q = warp & 3;
        for (int bk = warp >> 2; bk < g.nblk; bk += kThreads / 128) {
            const int f = bk * 128 + q * 32 + lane;
            for (int c0 = 0; c0 < g.NB; c0 += 16) {
                float v[16];
                umma::tmem_ld16(tH(c, bk) + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
                umma::tmem_wait_ld();
                if (f < D) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = c0 + i;
                        if (col < d) Hg[(size_t)f * d + col] = v[i];
                        else if (col == d) sg[f] = v[i];
                    }
                }
            }
        }
        for (int i = tid; i < Lmax; i += kThreads) S.pend[(size_t)st * Lmax + i] = (uint8_t)(i < pend_n ? lf[i] : 0);
        if (a.mode == 0) {
            for (int i = tid; i < lam; i += kThreads) {
                P.slotTok[(size_t)st * lam + i] = slotTok[i];
                P.slotVrow[(size_t)st * lam + i] = slotVrow[i];
            }
        }
    } else if (!ok) {
        if (tid == 0) {
            raise_error(S.err, ERR_TIMEOUT);
            umma::mbar_wait(&mbar, c.phase ^ 1u, kWaitNs);  // let an MMA still in flight drain
            for (int b = 0; b < 2; ++b)                      // and tile gathers still in flight
                if (tiss[b] != twait[b]) umma::mbar_wait(&tbar[b], twait[b] & 1u, kWaitNs);
        }
    }
    if (tid == 0) umma::bulk_wait_all();
    if (a.seg_done != nullptr && lead && tid == 0) {
        // gave up (or had no interval): count every segment not counted yet
        __threadfence();
        const int nseg = (a.n_int + a.seg_len - 1) / a.seg_len;
        for (int sg = seg_sig; sg < nseg; ++sg) atomicAdd(&a.seg_done[sg], 1);
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(c.tm, g.ncols);
    // no CTA leaves while a peer may still write into its shared memory (every CTA gets
    // here: all waits above are bounded)
    if (nc > 1) umma::cluster_sync();
}

}  // namespace

size_t chain_tc_smem_bytes(const Dims &dm) { return make_geo(dm).total; }

size_t snap_image_bytes(const Dims &dm)
{
    const Geo g = make_geo(dm);
    return (size_t)g.NB * g.FP * 2;
}

// CTAs per stream of a prefill chain. With few streams a cluster of up to 5 CTAs per
// stream shares the scoring, one SRE tile each or more (at most LOLA_CHAIN_CTAS CTAs in all,
// so that the attention keeps the other SMs; wider clusters measured slower: the key
// exchange grows with the width).
static int prefill_cluster(const Dims &dm)
{
    const int tiles = (dm.lam + dm.C + 127) / 128;   // SRE tiles of a full interval
    int nc = LOLA_CHAIN_CTAS / dm.ns;
    if (nc > tiles) nc = tiles;
    if (nc > 5) nc = 5;
    if (nc < 1) nc = 1;
    return nc;
}

int chain_tc_prefill_ctas(const Dims &dm) { return dm.ns * prefill_cluster(dm); }

void launch_chain_tc(const Dims &dm, const DevState &S, const PrefillScratch *P, const ChainArgs &a,
                     const CUtensorMap &phimap, const CUtensorMap &boxmap, cudaStream_t stream)
{
    KVSrc<bf16> src{(const bf16 *)S.KS, (const bf16 *)S.VS, (const bf16 *)S.KR, (const bf16 *)S.VR,
                    (const bf16 *)a.kin, (const bf16 *)a.vin, dm.lam, dm.R, a.n_call, dm.Hkv, dm.d,
                    a.call_start};
    const size_t smem = make_geo(dm).total;
    cudaFuncSetAttribute(chain_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    PrefillScratch Pv{};
    if (P) Pv = *P;
    const int nc = a.mode == 0 ? prefill_cluster(dm) : 1;
    if (nc == 1) {
        chain_tc_kernel<<<dm.ns, kThreads, smem, stream>>>(dm, S, Pv, a, src, 1, phimap, boxmap);
        return;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(dm.ns * nc), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, chain_tc_kernel, dm, S, Pv, a, src, nc, phimap, boxmap);
}

}  // namespace lola
