// Tensor-core feature map for bfloat16 rows (gist.science technical summary,
// "Probleemstelling": the low-rank positive feature map of the linear
// attention; this engine's form is phi(x) = [softmax(x W), softmax(-x W)]).
//
// One CTA walks tiles of 128 rows. A tile's rows are gathered into a K-major
// swizzled shared-memory tile (16-byte cp.async), Z = X W runs on the tensor
// cores into TMEM (Dh fp32 columns, W^T resident in shared memory as the
// K-major B operand), and one thread per row (its TMEM lane) takes the two
// softmaxes over the row's Dh values. The bf16 features are staged in shared
// memory and stored with coalesced 16-byte writes.
//
// Row sources: mode 0 = the virtual key rows of every stream (cache slots
// [0, nS), the ring, the call's tokens; see lola_internal.cuh), mode 1 = plain
// contiguous rows (queries).
#include "lola_internal.cuh"
#include "umma.cuh"

namespace lola {

namespace {

using bf16 = __nv_bfloat16;
constexpr int kThreads = 128;
constexpr uint64_t kWaitNs = 2000000000ull;

struct PGeo {
    int dp, Dh, D, ostride;
    uint32_t ncols;
    size_t off_w, off_out, off_rows, total;
};

__host__ __device__ inline size_t pal(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline PGeo make_pgeo(int d, int D)
{
    PGeo g{};
    g.dp = (d + 63) / 64 * 64;
    g.Dh = D / 2;
    g.D = D;
    g.ostride = D * 2 + 16;                               // staged output row (bytes, padded)
    g.ncols = g.Dh <= 32 ? 32 : g.Dh <= 64 ? 64 : g.Dh <= 128 ? 128 : 256;
    size_t o = (size_t)128 * g.dp * 2;                    // X tile
    g.off_w = pal(o, 1024);
    o = g.off_w + (size_t)g.Dh * g.dp * 2;                // W^T
    g.off_out = pal(o, 16);
    o = g.off_out + (size_t)128 * g.ostride;
    g.off_rows = pal(o, 16);
    o = g.off_rows + (size_t)128 * 16;                    // per-row source / destination
    g.total = o + 1024;
    return g;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    phi_tc_kernel(Dims dm, DevState S, KVSrc<bf16> src, int nS, int nvrows, long long nrows,
                  const bf16 *__restrict__ rows_in, bf16 *__restrict__ out)
{
    const int d = dm.d, D = dm.D;
    const PGeo g = make_pgeo(d, D);
    const int Dh = g.Dh;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lgd = __ffs(d >> 3) - 1;   // 16-byte chunks per input row (power of two)

    extern __shared__ uint8_t smraw[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    __shared__ int okflag;
    const uint32_t raw = umma::smem_u32(smraw);
    uint8_t *base = smraw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *sX = base, *sW = base + g.off_w, *sO = base + g.off_out;
    const bf16 **rin = (const bf16 **)(base + g.off_rows);
    bf16 **rout = (bf16 **)(base + g.off_rows + 128 * 8);

    if (tid == 0) umma::mbar_init(&mbar, 1);
    if (warp == 0) umma::tmem_alloc(&tslot, g.ncols);
    // W^T [Dh][d] as a K-major operand of Dh rows; with one W per kv-head, the CTAs of
    // grid row y take the rows of kv-head y
    const int hw = blockIdx.y;
    const bf16 *Wt = (const bf16 *)S.Wt + (size_t)hw * Dh * d;
    for (int e = tid; e < (Dh << lgd); e += kThreads) {
        const int r = e >> lgd, kc = e & ((1 << lgd) - 1);
        umma::cp_async16(sW + umma::kmajor_offset(r, kc * 8, Dh), Wt + (size_t)r * d + kc * 8);
    }
    umma::cp_async_commit();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tz = tslot;
    uint32_t phase = 0;
    const uint32_t idesc = umma::idesc_bf16(128, Dh, false, false);
    const int per_stream = nS + dm.R + (MODE == 0 ? src.n : 0);
    const bool by_head = gridDim.y > 1;
    // rows of this grid row: every row, or those of kv-head hw
    const long long nmine = !by_head ? nrows : MODE == 0 ? (long long)dm.B * per_stream : nrows / dm.Hq * dm.g;
    const long long ntiles = (nmine + 127) / 128;
    bool ok = true;

    for (long long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const long long r0 = tile * 128;
        const int nr = (int)min(128LL, nmine - r0);
        // this thread's row: where it comes from and where its features go
        {
            const long long rr = r0 + tid;
            long long gr = rr;
            if (by_head) {
                if (MODE == 0) gr = ((rr / per_stream) * dm.Hkv + hw) * per_stream + rr % per_stream;
                else gr = (rr / dm.g) * dm.Hq + (long long)hw * dm.g + rr % dm.g;
            }
            const bf16 *xi = nullptr;
            bf16 *yo = nullptr;
            if (tid < nr) {
                if (MODE == 0) {
                    const int st = (int)(gr / per_stream), i = (int)(gr % per_stream);
                    const int vrow = i < nS ? i : dm.lam + (i - nS);
                    xi = src.krow(st, vrow);
                    yo = out + ((size_t)st * nvrows + vrow) * D;
                } else {
                    xi = rows_in + (size_t)gr * d;
                    yo = out + (size_t)gr * D;
                }
            }
            rin[tid] = xi;
            rout[tid] = yo;
        }
        __syncthreads();
        for (int e = tid; e < (128 << lgd); e += kThreads) {
            const int r = e >> lgd, kc = e & ((1 << lgd) - 1);
            uint8_t *dst = sX + umma::kmajor_offset(r, kc * 8, 128);
            if (r < nr) umma::cp_async16(dst, rin[r] + kc * 8);
            else *(uint4 *)dst = make_uint4(0, 0, 0, 0);
        }
        umma::cp_async_commit();
        umma::cp_async_wait_all();
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t x0 = umma::smem_u32(sX), w0 = umma::smem_u32(sW);
            for (int ks = 0; ks < d / 16; ++ks)
                umma::mma_ss(tz, umma::kmajor_desc(x0, ks, 128), umma::kmajor_desc(w0, ks, Dh), idesc,
                             ks > 0 ? 1u : 0u);
            umma::mma_commit(&mbar);
            const bool fine = umma::mbar_wait_abortable(&mbar, phase, kWaitNs, S.err, ERR_TIMEOUT);
            if (!fine) raise_error(S.err, ERR_TIMEOUT);
            okflag = fine ? 1 : 0;
        }
        __syncthreads();
        phase ^= 1u;
        umma::fence_after_sync();
        if (!okflag) {
            ok = false;
            break;
        }
        // two softmaxes over this row's Dh values (three passes over TMEM)
        const uint32_t trow = tz + ((uint32_t)(warp * 32) << 16);
        float zmax = -INFINITY, zmin = INFINITY;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(trow + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                zmax = fmaxf(zmax, v[j]);
                zmin = fminf(zmin, v[j]);
            }
        }
        float sp = 0.f, sn = 0.f;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(trow + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                sp += __expf(v[j] - zmax);
                sn += __expf(zmin - v[j]);
            }
        }
        const float rp = 1.f / sp, rn = 1.f / sn;
        uint8_t *orow = sO + (size_t)tid * g.ostride;
        for (int c0 = 0; c0 < Dh; c0 += 16) {
            float v[16];
            umma::tmem_ld16(trow + (uint32_t)c0, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; j += 8) {
                uint4 pp, pn;
                pp.x = umma::pack_bf16x2(__expf(v[j] - zmax) * rp, __expf(v[j + 1] - zmax) * rp);
                pp.y = umma::pack_bf16x2(__expf(v[j + 2] - zmax) * rp, __expf(v[j + 3] - zmax) * rp);
                pp.z = umma::pack_bf16x2(__expf(v[j + 4] - zmax) * rp, __expf(v[j + 5] - zmax) * rp);
                pp.w = umma::pack_bf16x2(__expf(v[j + 6] - zmax) * rp, __expf(v[j + 7] - zmax) * rp);
                pn.x = umma::pack_bf16x2(__expf(zmin - v[j]) * rn, __expf(zmin - v[j + 1]) * rn);
                pn.y = umma::pack_bf16x2(__expf(zmin - v[j + 2]) * rn, __expf(zmin - v[j + 3]) * rn);
                pn.z = umma::pack_bf16x2(__expf(zmin - v[j + 4]) * rn, __expf(zmin - v[j + 5]) * rn);
                pn.w = umma::pack_bf16x2(__expf(zmin - v[j + 6]) * rn, __expf(zmin - v[j + 7]) * rn);
                *(uint4 *)(orow + (size_t)(c0 + j) * 2) = pp;
                *(uint4 *)(orow + (size_t)(Dh + c0 + j) * 2) = pn;
            }
        }
        umma::fence_before_sync();
        __syncthreads();
        // coalesced stores: consecutive threads write consecutive 16-byte pieces of a row
        const int cpr = D / 8;
        for (int e = tid; e < nr * cpr; e += kThreads) {
            const int r = e / cpr, c = e - r * cpr;
            *(uint4 *)(rout[r] + c * 8) = *(const uint4 *)(sO + (size_t)r * g.ostride + c * 16);
        }
        __syncthreads();
    }
    umma::cp_async_wait_all();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tz, g.ncols);
}

dim3 phi_tc_grid(long long nrows, const Dims &dm)
{
    nrows /= dm.nW;
    const PGeo g = make_pgeo(dm.d, dm.D);
    int per_sm = (int)((228 * 1024) / (g.total + 1024));
    if (per_sm < 1) per_sm = 1;
    if (per_sm > 4) per_sm = 4;
    long long tiles = (nrows + 127) / 128;
    long long grid = 148LL * per_sm / dm.nW;
    if (grid > tiles) grid = tiles;
    return dim3((unsigned)(grid < 1 ? 1 : grid), (unsigned)dm.nW);
}

}  // namespace

size_t phi_tc_smem_bytes(const Dims &dm) { return make_pgeo(dm.d, dm.D).total; }

void launch_phi_kv_tc(const Dims &dm, const DevState &S, const void *kin, long long call_start, int n,
                      int nvrows, void *phi_out, int nS, cudaStream_t stream)
{
    KVSrc<bf16> src{(const bf16 *)S.KS, (const bf16 *)S.VS, (const bf16 *)S.KR, (const bf16 *)S.VR,
                    (const bf16 *)kin, nullptr, dm.lam, dm.R, n, dm.Hkv, dm.d, call_start};
    const long long rows = (long long)dm.ns * (nS + dm.R + n);
    const size_t smem = make_pgeo(dm.d, dm.D).total;
    static size_t attr = 0;   // largest opt-in set so far
    if (smem > attr) {
        cudaFuncSetAttribute(phi_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        attr = smem;
    }
    phi_tc_kernel<0><<<phi_tc_grid(rows, dm), kThreads, smem, stream>>>(dm, S, src, nS, nvrows, rows,
                                                                        nullptr, (bf16 *)phi_out);
}

void launch_phi_q_tc(const Dims &dm, const DevState &S, const void *q, long long rows, void *phi_out,
                     cudaStream_t stream)
{
    KVSrc<bf16> src{};
    const size_t smem = make_pgeo(dm.d, dm.D).total;
    static size_t attr = 0;   // largest opt-in set so far
    if (smem > attr) {
        cudaFuncSetAttribute(phi_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        attr = smem;
    }
    phi_tc_kernel<1><<<phi_tc_grid(rows, dm), kThreads, smem, stream>>>(dm, S, src, 0, 0, rows,
                                                                        (const bf16 *)q, (bf16 *)phi_out);
}

}  // namespace lola
