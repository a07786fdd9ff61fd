// Internal definitions shared by the LoLA CUDA kernels (sm_100a).
//
// One "stream" is one (batch, kv-head) pair; every piece of state is per
// stream and read by the n_q_heads / n_kv_heads query heads of its group.
//
// Virtual rows. Keys and values that a prefill call touches live in three
// places: the state's sparse-cache slots, the state's window ring, and the
// caller's k/v buffers. The kernels address them through one row index per
// stream:  [0, lam)            cache slot i
//          [lam, lam + R)      ring slot (token mod R; R is a power of two)
//          [lam + R, lam+R+n)  token call_start + (row - lam - R) of the call
// phi(k) scratch is laid out over the same rows. Its rows [0, lam) always hold
// phi of the pair currently in each cache slot (the tensor-core chain rewrites
// a slot's row when a new pair takes the slot), so the chain loads the cached
// candidates as contiguous 128-row blocks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lola {

enum : int { ERR_BOUNDS = 1, ERR_TIMEOUT = 2 };
constexpr int kMaxSegments = 64;   // prefill segments per call, at most

struct Dims {
    int B, Hq, Hkv, g, d, D, Dh, eta, lam, C, Cdec, R, Lmax, ns, dtype;
    int Nmax, mmax;   // prefill scratch capacity: tokens per call, intervals per call
    int nsplit;       // decode: partial records per stream (CTAs, or warp ranges)
    int dec_nw;       // decode: warps per CTA
    int dec_nst;      // decode: staging buffers per warp
    int dec_sb;       // decode: bytes per staging buffer
    int dec_tma;      // decode (bf16): key/value chunks arrive by tiled TMA loads (128 B swizzle)
    int dec_minper;   // decode (bf16): fewest work items per warp (fewer for few streams)
    int tc_chain;     // 1: tensor-core chain (bf16), 0: SIMT chain
    int tc_attn;      // 1: tensor-core prefill attention (bf16, head_dim % 64 == 0)
    int attn_ws;      // 1: its warp-specialised form (feature half a multiple of 64, 128 % g == 0)
    int scorer;       // cache scoring: 0 SRE, 1 attention weight, 2 softmax-approximation error, 3 recency
    int nW;           // feature-map matrices: 1 (shared) or Hkv (one per kv-head)
    float eps;
};

// Persistent state (device pointers into the caller's workspace).
struct DevState {
    float *H;          // [ns][D][d]   fp32 linear-attention state
    float *s;          // [ns][D]      fp32 normaliser
    void *KS, *VS;     // [ns][lam][d] sparse-cache keys / values (dtype)
    int *idxS;         // [ns][lam]    token index per cache slot, -1 = empty
    void *KR, *VR;     // [ns][R][d]   window ring (slot = token mod R)
    uint8_t *pend;     // [ns][Lmax]   1 = leaving pair of the last interval that is folded
    float *W;          // [nW][d][Dh]  feature-map matrices (one per kv-head, or one shared), fp32 copy
    void *Wt;          // [nW][Dh][d]  W transposed, in the input dtype (tensor-core operand)
    void *WtImg;       // [nW][Dh * d] bfloat16 W^T as a K-major 128-byte-swizzled operand image
                       //              (Dh rows, d columns; bfloat16 states with d % 64 == 0)
    int *err;          // [4]          device error words
    // decode scratch (phi buffers hold the input dtype)
    void *phiV;        // [ns][lam + R][D] phi of cache slots and ring rows (decode interval)
    float *part;       // [ns][nsplit][g][2d + 4] partials of the warps / CTAs sharing a stream
    float *phiQd;      // [B][Hq][D]   fp32 phi(q) of the decode step (bfloat16 path)
    int *dec_cnt;      // [ns] finished decode CTAs per stream (reset by the last one)
    int *seg_done;     // [kMaxSegments] prefill: streams whose chain has finished a segment of
                       //   the call, counted up across calls (the attention of a segment waits
                       //   for its count with a stream memory operation)
};

// Per-prefill-call scratch.
struct PrefillScratch {
    void *phiK;        // [ns][lam + R + Nmax][D]  (input dtype)
    void *phiQ;        // [B][Nmax][Hq][D]         (input dtype)
    void *snapImg;     // [ns][mmax][NB x FP] bf16 K-major image of [H'|s'] (tensor-core path)
    float *snapH;      // [ns][mmax][D][d]  H' of each interval (after the cache eviction fold)
    float *snapS;      // [ns][mmax][D]
    int *logTok;       // [ns][mmax][lam]   kept set of each interval (token)
    int *logVrow;      // [ns][mmax][lam]   kept set of each interval (virtual row)
    int *logCount;     // [ns][mmax]
    uint8_t *logLf;    // [ns][mmax][Cmax]  leaving-pair fate per interval, 1 = folded
    int *slotTok;      // [ns][lam]         slot contents at the end of the call
    int *slotVrow;     // [ns][lam]
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x)
{
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

// Key/value row addressing over virtual rows (see the file comment).
template <typename T> struct KVSrc {
    const T *KS, *VS;    // [ns][lam][d]
    const T *KR, *VR;    // [ns][R][d]
    const T *kin, *vin;  // [B][n][Hkv][d] (prefill call), may be null
    int lam, R, n, Hkv, d;
    long long call_start; // token index of call row 0

    __device__ __forceinline__ const T *row(const T *cache, const T *ring, const T *in, int st,
                                            int vrow) const
    {
        if (vrow < lam) return cache + ((size_t)st * lam + vrow) * d;
        if (vrow < lam + R) return ring + ((size_t)st * R + (vrow - lam)) * d;
        const int b = st / Hkv, hk = st % Hkv;
        return in + (((size_t)b * n + (vrow - lam - R)) * Hkv + hk) * d;
    }
    __device__ __forceinline__ const T *krow(int st, int vrow) const { return row(KS, KR, kin, st, vrow); }
    __device__ __forceinline__ const T *vrow(int st, int vrow) const { return row(VS, VR, vin, st, vrow); }
    // virtual row of a window/call token (never a cache slot)
    __device__ __forceinline__ int tok2vrow(long long tok) const
    {
        if (kin != nullptr && tok >= call_start) return lam + R + (int)(tok - call_start);
        return lam + (int)(tok & (R - 1));  // R is a power of two
    }
};

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_min(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// The feature-map matrix of kv-head hk (W: [nW][d][Dh]).
__device__ __forceinline__ const float *w_of(const Dims &dm, const float *W, int hk)
{
    return dm.nW > 1 ? W + (size_t)hk * dm.d * dm.Dh : W;
}

// phi(x) = [softmax(x W), softmax(-x W)] of one row, computed by one warp. W (fp32, [d][Dh]) sits in shared memory; lane l owns
// features l, l + 32, ... The row max / min shift is exact in real arithmetic.
template <typename T, typename O>
__device__ __forceinline__ void phi_row_warp(const T *__restrict__ x, const float *__restrict__ Ws,
                                             float *__restrict__ xs, int d, int Dh,
                                             O *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    for (int a = lane; a < d; a += 32) xs[a] = to_f<T>(x[a]);
    __syncwarp();
    float z[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) z[u] = 0.f;
    for (int a = 0; a < d; ++a) {
        const float xa = xs[a];
        const float *wr = Ws + (size_t)a * Dh;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = lane + 32 * u;
            if (i < Dh) z[u] = fmaf(xa, wr[i], z[u]);
        }
    }
    float zmax = -INFINITY, zmin = INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (lane + 32 * u < Dh) {
            zmax = fmaxf(zmax, z[u]);
            zmin = fminf(zmin, z[u]);
        }
    }
    zmax = warp_max(zmax);
    zmin = warp_min(zmin);
    float ep[4], en[4], sp = 0.f, sn = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const bool ok = lane + 32 * u < Dh;
        ep[u] = ok ? __expf(z[u] - zmax) : 0.f;
        en[u] = ok ? __expf(zmin - z[u]) : 0.f;
        sp += ep[u];
        sn += en[u];
    }
    sp = warp_sum(sp);
    sn = warp_sum(sn);
    const float rp = 1.f / sp, rn = 1.f / sn;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = lane + 32 * u;
        if (i < Dh) {
            out[i] = from_f<O>(ep[u] * rp);
            out[Dh + i] = from_f<O>(en[u] * rn);
        }
    }
    __syncwarp();
}

__device__ __forceinline__ void raise_error(int *err, int code)
{
    if (err) atomicOr(err, code);
}

// CTA-uniform check at kernel entry: an earlier kernel of this state recorded an
// error. Kernels that read the per-interval logs of the chain skip their work then
// (after a chain gave up, those logs may be incomplete); lola_sync reports the
// error and clears the word.
__device__ __forceinline__ bool cta_error_pending(const int *err)
{
    __shared__ int flag;
    if (threadIdx.x == 0) flag = *(const volatile int *)err;
    __syncthreads();
    return flag != 0;
}

// ---- host launch wrappers (defined in the .cu files) ----
void launch_init_state(const Dims &dm, const DevState &S, const void *W, cudaStream_t stream);
void launch_phi_kv(const Dims &dm, const DevState &S, const void *kin, long long call_start,
                   int n, int nvrows, int row_begin_call, void *phi_out, int nS,
                   cudaStream_t stream);
void launch_phi_q(const Dims &dm, const float *W, const void *q, long long rows, void *phi_out,
                  cudaStream_t stream);
// bfloat16 tensor-core versions of the two above
void launch_phi_kv_tc(const Dims &dm, const DevState &S, const void *kin, long long call_start, int n,
                      int nvrows, void *phi_out, int nS, cudaStream_t stream);
void launch_phi_q_tc(const Dims &dm, const DevState &S, const void *q, long long rows, void *phi_out,
                     cudaStream_t stream);
size_t phi_tc_smem_bytes(const Dims &dm);

struct ChainArgs {
    int mode;               // 0 = prefill call, 1 = decode interval
    long long pos0;         // first token of the first interval
    int n_int, ilen;        // intervals and their length
    long long call_start;   // prefill: token of call row 0
    int n_call;             // prefill: tokens in the call
    const void *kin, *vin;  // prefill: call k/v
    int nS0;                // cache occupancy before the first interval
    long long pend_lo;      // pending leaving range of the previous interval
    int pend_n;
    long long iglob0;       // interval counter of the first interval
    const void *phi;        // [ns][nvrows][D] (input dtype)
    int nvrows;
    int32_t *sel_log;       // test hook, may be null
    long long sel_cap;
    const int32_t *ovr;     // test hook, may be null
    long long ovr_n;
    const void *qin;        // queries holding every interval's first query (alternative scorers):
    long long q_start;      //   [B][q_n][Hq][d], row 0 = token q_start
    int q_n;
    unsigned long long inject_ns;   // test hook: > 0 makes the first interval wait this long on an
                                    // mbarrier nothing arrives at (the wait runs out: timeout)
    float *score_sre;       // test hook, may be null: SRE of every candidate
    int32_t *score_tok;     //   and its token, [interval][ns][lam + Lmax] (candidate order)
    long long score_cap;
    int snap_f32;           // prefill: also write fp32 (H', s') snapshots
    int ci0;                // prefill: index of the first interval within the call
    int *seg_done;          // prefill, may be null: the lead CTA of every stream adds 1 to
    int seg_len;            //   seg_done[s] once it has finished the intervals of segment s
                            //   (seg_len intervals each; the call's logs and snapshots of them
                            //   are written and visible), and to every segment left when it
                            //   gives up, so that no wait for a count is left without it
    int cont;               // prefill: the call's earlier intervals ran in an earlier launch
                            // (slot contents come from the scratch, not the state)
};
// phimap / boxmap: row maps of a.phi as [ns * a.nvrows][D] with 1-row / 128-row boxes
void launch_chain_tc(const Dims &dm, const DevState &S, const PrefillScratch *P, const ChainArgs &a,
                     const CUtensorMap &phimap, const CUtensorMap &boxmap, cudaStream_t stream);
size_t chain_tc_smem_bytes(const Dims &dm);
size_t attn_tc_smem_bytes(const Dims &dm);
size_t snap_image_bytes(const Dims &dm);
void launch_chain(const Dims &dm, const DevState &S, const PrefillScratch *P, const ChainArgs &a,
                  cudaStream_t stream);

struct AttnArgs {
    long long pos0;         // first token of the call
    int m;                  // chunks in this launch
    int ci0;                // index of this launch's first chunk within the call
    int n_call;
    const void *q, *kin, *vin;
    void *out;
};
void launch_attn_prefill(const Dims &dm, const DevState &S, const PrefillScratch &P,
                         const AttnArgs &a, cudaStream_t stream);
void launch_attn_tc(const Dims &dm, const DevState &S, const PrefillScratch &P, const AttnArgs &a,
                    cudaStream_t stream);
// Warp-specialised tensor-core prefill attention (bfloat16, two query tiles per CTA).
// Tensor maps of one call: q [B * n][Hq][d] (boxes of 128 query rows of one
// kv-head group), k and v [B * n][Hkv][d] (boxes of 64 tokens of one kv-head),
// and the phi rows [ns * (lam + R + Nmax)][D] (64-row boxes).
struct AttnMaps {
    CUtensorMap q, k, v, phik;
};
bool attn_ws_supported(const Dims &dm);
size_t attn_ws_smem_bytes(const Dims &dm);
bool make_attn_maps(const Dims &dm, const AttnArgs &a, const void *phiK, AttnMaps *maps);
void launch_attn_ws(const Dims &dm, const DevState &S, const PrefillScratch &P, const AttnArgs &a,
                    const AttnMaps &maps, cudaStream_t stream);
void launch_finalize_prefill(const Dims &dm, const DevState &S, const PrefillScratch &P,
                             const void *kin, const void *vin, long long call_start, int n,
                             int nK, cudaStream_t stream);

// Tiled TMA descriptors of the cache and ring key/value arrays, 3-D
// [stream][row][head_dim] with 32-row x 64-element boxes and 128-byte swizzle.
struct DecMaps {
    CUtensorMap ks, vs, kr, vr;
};

// Row map of a bfloat16 array [rows][cols]: boxes of box_rows x 64 columns,
// 128-byte swizzle, zero fill past the extent (box_rows 1: tile::gather4 loads);
// false if encoding fails.
bool make_row_map(CUtensorMap *m, const void *base, unsigned long long rows, int cols, int box_rows);
// 3-D map of a bfloat16 array [d2][d1][d0] with 64 x box1 x box2 boxes, 128-byte
// swizzle, zero fill past the extent; false if encoding fails.
bool make_map_3d(CUtensorMap *m, const void *base, int d0, int d1, unsigned long long d2, int box1, int box2);

struct DecodeArgs {
    long long pos;          // token index of this step
    long long t0;           // start of the open interval
    int nS;                 // cache occupancy during the interval
    long long L_lo;         // leaving range of the open interval [L_lo, L_hi)
    long long L_hi;
    const void *q, *k, *v;
    void *out;
    unsigned long long inject_ns;   // test hook: > 0 makes the streaming kernel's first warp wait
                                    // this long on an mbarrier nothing arrives at (timeout)
    int state_ahead;        // 1: the state already holds the open interval's folded leaving pairs
                            // (tensor-core chain); 0: they fold at the next interval's start
};
// Decode launch shape: splits per stream, warps per CTA, staging buffers and
// their size (fills dm.nsplit, dec_nw, dec_nst, dec_sb); returns false if no
// shape fits in shared memory.
bool decode_plan(Dims *dm);
size_t decode_smem_bytes(const Dims &dm);
// with_phi: also compute phi(k) of the appended token into the phi rows.
void launch_decode_append(const Dims &dm, const DevState &S, const void *k, const void *v,
                          long long pos, int with_phi, cudaStream_t stream);
// do_append: the kernel also appends the step's k, v (and phi(k)) to the window ring.
void launch_decode_attn(const Dims &dm, const DevState &S, const DecodeArgs &a, int do_append,
                        const DecMaps *maps, cudaStream_t stream);
// Encodes the four maps for the state's buffers; false if the driver call fails.
bool make_decode_maps(const Dims &dm, const DevState &S, DecMaps *maps);
void launch_get_indices(const Dims &dm, const DevState &S, int nS, int32_t *idx, int32_t *cnt,
                        cudaStream_t stream);

}  // namespace lola
