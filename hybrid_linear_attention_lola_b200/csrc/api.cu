// Host side of the C ABI declared in include/lola.h: argument checks, the
// workspace layout, and the order in which one prefill call or decode step
// enqueues its kernels on the caller's stream.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/lola.h"
#include "lola_internal.cuh"

namespace lola {
size_t chain_smem_bytes(const Dims &dm);
size_t attn_smem_bytes(const Dims &dm);
int chain_tc_prefill_ctas(const Dims &dm);   // CTAs (SMs) a tensor-core prefill chain occupies
}

struct lola_state {
    lola_config cfg;
    lola::Dims dm;
    lola::DevState S;
    lola::PrefillScratch P;
    void *ws;
    size_t ws_bytes;
    long long pos;           // tokens processed per sequence
    long long interval_end;  // end of the open decode interval (== pos when none is open)
    long long t0_open;       // start of the open (or last) decode interval
    int nS;                  // cache occupancy (identical for every stream)
    long long pend_lo;       // leaving pairs of the last interval: [pend_lo, pend_lo + pend_n)
    int pend_n;
    long long n_int;         // update intervals run since init/reset
    bool phiV_valid;         // phi rows of the cache slots and the ring are current
    // prefill segments: chain on a high-priority library stream, the attention of even
    // segments on the caller's stream and of odd segments on a second library stream, so
    // that a segment's last partial wave of CTAs overlaps the next segment's first
    static constexpr int kMaxSeg = lola::kMaxSegments;
    bool overlap;                    // the streams and events of segmented prefill exist
    int sms;                         // SMs of the state's device
    int sched_mode;                  // lola_schedule of the following prefill calls
    int seg_user;                    // intervals per segment asked for (0: the mode's default)
    cudaStream_t chain_stream;
    cudaStream_t attn_stream;
    cudaEvent_t ev_fork;
    cudaEvent_t ev_attn;             // the second attention stream's work of a call is done
    cudaEvent_t ev_seg[kMaxSeg];
    // one chain launch per call: the attention of segment s waits (stream memory
    // operation) until seg_done[s] reaches seg_expect[s], the streams' running count
    bool seg_wait;
    uint32_t seg_expect[lola::kMaxSegments];
    // prefill from host memory: copy streams (host to device, device to host) and the
    // events of the two staging slots (created at the first such call)
    cudaStream_t h2d_stream, d2h_stream;
    cudaEvent_t ev_h2d[2], ev_comp[2], ev_d2h[2], ev_host;
    lola::DecMaps maps;              // TMA descriptors of the cache / ring arrays (bf16 decode)
    CUtensorMap phik_map, phik_box;  // row maps (1-row and 128-row boxes) of the prefill and the
    CUtensorMap phiv_map, phiv_box;  // decode phi rows (tensor-core chain)
    int32_t *sel_log;
    long long sel_cap;
    const int32_t *ovr;
    long long ovr_n;
    float *score_sre;
    int32_t *score_tok;
    long long score_cap;
    int inject_where;                // fault-injection hook (one shot): 1 chain, 2 decode streaming kernel
    unsigned long long inject_ns;
    // timing hook
    bool timing;
    struct Mark { int phase; cudaEvent_t a, b; };
    std::vector<Mark> marks;
    std::vector<cudaEvent_t> pool;
};

namespace {

using lola::Dims;

std::atomic<long long> g_launches{0};
void counted(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

enum Phase { PH_PHI = 0, PH_CHAIN, PH_ATTN, PH_FINAL, PH_APPEND, PH_UPDATE, PH_DECODE, PH_RESET };

cudaEvent_t take_event(lola_state *st)
{
    if (!st->pool.empty()) {
        cudaEvent_t e = st->pool.back();
        st->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets a group of launches with events when the timing hook is on.
struct PhaseScope {
    lola_state *st;
    int phase;
    cudaStream_t stream;
    cudaEvent_t a = nullptr;
    PhaseScope(lola_state *s, int ph, cudaStream_t strm) : st(s), phase(ph), stream(strm)
    {
        if (st->timing) {
            a = take_event(st);
            cudaEventRecord(a, stream);
        }
    }
    ~PhaseScope()
    {
        if (st->timing && a) {
            cudaEvent_t b = take_event(st);
            cudaEventRecord(b, stream);
            st->marks.push_back({phase, a, b});
        }
    }
};

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

lola_status derive_dims(const lola_config *c, Dims *dm)
{
    if (!c) return LOLA_ERR_INVALID_ARG;
    if (c->dtype != LOLA_F32 && c->dtype != LOLA_BF16) return LOLA_ERR_DTYPE;
    if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads)
        return LOLA_ERR_INVALID_ARG;
    const int g = c->n_q_heads / c->n_kv_heads;
    if (g > 8) return LOLA_ERR_INVALID_ARG;
    if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return LOLA_ERR_INVALID_ARG;
    if (c->feat_dim % 32 != 0 || c->feat_dim < 32 || c->feat_dim > 256) return LOLA_ERR_INVALID_ARG;
    if (c->window < 0 || c->window > 65536) return LOLA_ERR_INVALID_ARG;
    if (c->lambda_ < 0 || c->lambda_ > 4096) return LOLA_ERR_INVALID_ARG;
    if (c->chunk < 1 || c->chunk > 256) return LOLA_ERR_INVALID_ARG;
    if (c->decode_interval < 1 || c->decode_interval > 256 || c->decode_interval > c->window + 1)
        return LOLA_ERR_INVALID_ARG;
    if (!(c->eps >= 0.f)) return LOLA_ERR_INVALID_ARG;
    if (c->scorer < LOLA_SCORE_SRE || c->scorer > LOLA_SCORE_RECENCY) return LOLA_ERR_INVALID_ARG;
    if (c->w_per_kv_head != 0 && c->w_per_kv_head != 1) return LOLA_ERR_INVALID_ARG;
    const int nmax = c->max_prefill_tokens > 0 ? c->max_prefill_tokens : c->chunk;
    if (nmax % c->chunk != 0) return LOLA_ERR_INVALID_ARG;
    dm->B = c->batch;
    dm->Hq = c->n_q_heads;
    dm->Hkv = c->n_kv_heads;
    dm->g = g;
    dm->d = c->head_dim;
    dm->D = c->feat_dim;
    dm->Dh = c->feat_dim / 2;
    dm->eta = c->window;
    dm->lam = c->lambda_;
    dm->C = c->chunk;
    dm->Cdec = c->decode_interval;
    dm->Lmax = c->chunk > c->decode_interval ? c->chunk : c->decode_interval;
    // ring slots: a power of two >= window + longest interval + 1 (slot = token & (R - 1))
    dm->R = 1;
    while (dm->R < c->window + dm->Lmax + 1) dm->R <<= 1;
    dm->ns = c->batch * c->n_kv_heads;
    dm->dtype = c->dtype;
    dm->Nmax = nmax;
    dm->mmax = nmax / c->chunk;
    dm->eps = c->eps;
    dm->scorer = c->scorer;
    dm->nW = c->w_per_kv_head ? c->n_kv_heads : 1;
    if (!lola::decode_plan(dm)) return LOLA_ERR_INVALID_ARG;
    // the tensor-core chain selects into a cache (lambda = 0 runs on the SIMT chain) and
    // holds the state image as an N-contiguous operand of whole 64-column atoms
    // It folds every unkept pair of an interval at once, so the prefill attention that
    // reads its snapshots is the tensor-core one (it takes the state at the interval's
    // end): the two run together or not at all.
    dm->tc_chain = (c->dtype == LOLA_BF16 && dm->lam > 0 && dm->d % 64 == 0 &&
                    lola::chain_tc_smem_bytes(*dm) <= 227 * 1024 && lola::attn_tc_smem_bytes(*dm) <= 227 * 1024)
                       ? 1 : 0;
    if (!dm->tc_chain && lola::chain_smem_bytes(*dm) > 227 * 1024) return LOLA_ERR_INVALID_ARG;
    dm->tc_attn = dm->tc_chain;
    dm->attn_ws = dm->tc_attn && lola::attn_ws_supported(*dm) ? 1 : 0;
    if (lola::attn_smem_bytes(*dm) > 227 * 1024) return LOLA_ERR_INVALID_ARG;
    if (c->dtype == LOLA_BF16 && lola::phi_tc_smem_bytes(*dm) > 227 * 1024) return LOLA_ERR_INVALID_ARG;
    return LOLA_OK;
}

size_t elem_bytes(const Dims &dm) { return dm.dtype == LOLA_F32 ? 4 : 2; }

// Carves the workspace; with base == nullptr only the size is computed.
size_t layout(const Dims &dm, char *base, lola::DevState *S, lola::PrefillScratch *P)
{
    size_t off = 0;
    auto take = [&](size_t bytes) -> void * {
        void *p = base ? base + off : nullptr;
        off = align_up(off + bytes);
        return p;
    };
    const size_t e = elem_bytes(dm);
    const size_t ns = dm.ns;
    lola::DevState s{};
    s.err = (int *)take(16);
    s.H = (float *)take(ns * dm.D * dm.d * 4);
    s.s = (float *)take(ns * dm.D * 4);
    s.KS = take(ns * dm.lam * dm.d * e);
    s.VS = take(ns * dm.lam * dm.d * e);
    s.idxS = (int *)take(ns * dm.lam * 4);
    s.KR = take(ns * dm.R * dm.d * e);
    s.VR = take(ns * dm.R * dm.d * e);
    s.pend = (uint8_t *)take(ns * dm.Lmax);
    s.W = (float *)take((size_t)dm.nW * dm.d * dm.Dh * 4);
    s.Wt = take((size_t)dm.nW * dm.d * dm.Dh * e);
    s.WtImg = (dm.dtype == LOLA_BF16 && dm.d % 64 == 0) ? take((size_t)dm.nW * dm.d * dm.Dh * 2) : nullptr;
    s.phiV = take(ns * (dm.lam + dm.R) * dm.D * e);
    s.part = (float *)take(ns * dm.nsplit * dm.g * (2 * dm.d + 4) * 4);
    s.phiQd = (float *)take(dm.dtype == LOLA_BF16 ? (size_t)dm.B * dm.Hq * dm.D * 4 : 0);
    s.dec_cnt = (int *)take(ns * 4);
    s.seg_done = (int *)take(lola::kMaxSegments * 4);
    lola::PrefillScratch p{};
    const size_t nv = (size_t)dm.lam + dm.R + dm.Nmax;
    p.phiK = take(ns * nv * dm.D * e);
    p.phiQ = dm.tc_attn ? nullptr : take((size_t)dm.B * dm.Nmax * dm.Hq * dm.D * e);
    p.snapH = (float *)take(dm.tc_attn ? 0 : ns * dm.mmax * dm.D * dm.d * 4);
    p.snapS = (float *)take(dm.tc_attn ? 0 : ns * dm.mmax * dm.D * 4);
    p.snapImg = dm.tc_chain ? take(ns * dm.mmax * lola::snap_image_bytes(dm)) : nullptr;
    p.logTok = (int *)take(ns * dm.mmax * dm.lam * 4);
    p.logVrow = (int *)take(ns * dm.mmax * dm.lam * 4);
    p.logCount = (int *)take(ns * dm.mmax * 4);
    p.logLf = (uint8_t *)take(ns * dm.mmax * dm.Lmax);
    p.slotTok = (int *)take(ns * dm.lam * 4);
    p.slotVrow = (int *)take(ns * dm.lam * 4);
    if (S) *S = s;
    if (P) *P = p;
    return off;
}

lola_status check_launch()
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        fprintf(stderr, "lola: CUDA error: %s\n", cudaGetErrorString(e));
        return LOLA_ERR_CUDA;
    }
    return LOLA_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

void reset_host(lola_state *st)
{
    st->pos = 0;
    st->interval_end = 0;
    st->t0_open = 0;
    st->nS = 0;
    st->pend_lo = 0;
    st->pend_n = 0;
    st->n_int = 0;
    st->phiV_valid = false;
}

// The armed fault-injection wait limit if it targets `where` (then disarmed), else 0.
unsigned long long take_injection(lola_state *st, int where)
{
    if (st->inject_where != where) return 0;
    st->inject_where = 0;
    return st->inject_ns;
}

// Host mirror of one interval's bookkeeping (identical for every stream).
void advance_interval(lola_state *st, long long t0, int len)
{
    const long long t1 = t0 + len;
    long long lo = t0 - st->dm.eta;
    if (lo < 0) lo = 0;
    long long hi = t1 - st->dm.eta;
    if (hi < lo) hi = lo;
    const int nL = (int)(hi - lo);
    const int nQ = st->nS + nL;
    st->nS = nQ < st->dm.lam ? nQ : st->dm.lam;
    st->pend_lo = lo;
    st->pend_n = nL;
    st->n_int += 1;
}

// One decode step. `part` receives the split partials of the decode attention.
lola_status decode_step_impl(lola_state *st, const void *q, const void *k, const void *v, void *out,
                             void *cuda_stream, float *part, float *phiq)
{
    if (!st || !q || !k || !v || !out) return LOLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return LOLA_ERR_INVALID_ARG;
    const Dims &dm = st->dm;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    const long long pos = st->pos;
    int do_append = 1;
    if (pos == st->interval_end) {
        // an update interval opens: the new pair joins the ring first (it may
        // already be a leaving pair), then score / select / fold
        {
            PhaseScope ps(st, PH_APPEND, stream);
            lola::launch_decode_append(dm, st->S, k, v, pos, st->phiV_valid ? 1 : 0, stream);
            counted(1);
        }
        if (check_launch() != LOLA_OK) return LOLA_ERR_CUDA;
        do_append = 0;
        PhaseScope ps(st, PH_UPDATE, stream);
        if (!st->phiV_valid) {
            if (dm.dtype == LOLA_BF16)
                lola::launch_phi_kv_tc(dm, st->S, nullptr, 0, 0, dm.lam + dm.R, st->S.phiV, st->nS, stream);
            else
                lola::launch_phi_kv(dm, st->S, nullptr, 0, 0, dm.lam + dm.R, 0, st->S.phiV, st->nS, stream);
            counted(1);
        }
        lola::ChainArgs ca{};
        ca.mode = 1;
        ca.pos0 = pos;
        ca.n_int = 1;
        ca.ilen = dm.Cdec;
        ca.call_start = 0;
        ca.n_call = 0;
        ca.kin = nullptr;
        ca.vin = nullptr;
        ca.nS0 = st->nS;
        ca.pend_lo = st->pend_lo;
        ca.pend_n = st->pend_n;
        ca.iglob0 = st->n_int;
        ca.phi = st->S.phiV;
        ca.nvrows = dm.lam + dm.R;
        ca.qin = q;          // the step's query is the interval's first
        ca.q_start = pos;
        ca.q_n = 1;
        ca.sel_log = st->sel_log;
        ca.sel_cap = st->sel_cap;
        ca.ovr = st->ovr;
        ca.ovr_n = st->ovr_n;
        ca.score_sre = st->score_sre;
        ca.score_tok = st->score_tok;
        ca.score_cap = st->score_cap;
        ca.inject_ns = take_injection(st, 1);
        if (dm.tc_chain) lola::launch_chain_tc(dm, st->S, nullptr, ca, st->phiv_map, st->phiv_box, stream);
        else lola::launch_chain(dm, st->S, nullptr, ca, stream);
        counted(1);
        if (check_launch() != LOLA_OK) return LOLA_ERR_CUDA;
        st->phiV_valid = true;
        advance_interval(st, pos, dm.Cdec);
        st->t0_open = pos;
        st->interval_end = pos + dm.Cdec;
    }
    lola::DecodeArgs da{};
    da.pos = pos;
    da.t0 = st->t0_open;
    da.nS = st->nS;
    da.L_lo = st->pend_lo;
    da.L_hi = st->pend_lo + st->pend_n;
    da.q = q;
    da.k = k;
    da.v = v;
    da.out = out;
    da.inject_ns = dm.dtype == LOLA_BF16 ? take_injection(st, 2) : 0;
    da.state_ahead = dm.tc_chain;
    lola::DevState Sx = st->S;
    Sx.part = part;
    Sx.phiQd = phiq;
    {
        PhaseScope ps(st, PH_DECODE, stream);
        lola::launch_decode_attn(dm, Sx, da, do_append, dm.dec_tma ? &st->maps : nullptr, stream);
        counted(1);
    }
    st->pos = pos + 1;
    return check_launch();
}

}  // namespace

namespace {

// cuStreamWaitValue32: a stream waits until a 32-bit word in device memory reaches a
// value (no kernel spins; the stream's front end holds the next work)
using WaitValueFn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
WaitValueFn wait_value_fn()
{
    static WaitValueFn fn = []() -> WaitValueFn {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuStreamWaitValue32", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return (WaitValueFn)f;
    }();
    return fn;
}

// Staging of lola_prefill_host: two slots, each holding a piece's q, k, v and out.
struct HostSlot {
    size_t q, kv, total;   // bytes of the q (and out) piece, of a k (or v) piece, of a slot
};
HostSlot host_slot(const Dims &dm, int64_t piece)
{
    HostSlot h;
    const size_t e = elem_bytes(dm);
    h.q = (size_t)dm.B * piece * dm.Hq * dm.d * e;
    h.kv = (size_t)dm.B * piece * dm.Hkv * dm.d * e;
    h.total = 2 * align_up(h.q) + 2 * align_up(h.kv);
    return h;
}

bool make_host_streams(lola_state *st)
{
    if (st->h2d_stream != nullptr) return true;
    bool ok = cudaStreamCreateWithFlags(&st->h2d_stream, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&st->d2h_stream, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&st->ev_host, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
        ok = cudaEventCreateWithFlags(&st->ev_h2d[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&st->ev_comp[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&st->ev_d2h[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        // the handles created so far stay valid until lola_free_state destroys them
        cudaGetLastError();
        return false;
    }
    return true;
}

// Configs whose prefill runs in overlapped segments: the tensor-core chain and attention,
// more than one interval per call.
bool segmented_prefill(const Dims &dm) { return dm.tc_chain && dm.tc_attn && dm.mmax > 1; }

// The schedule of a segmented prefill call of m intervals (mode and seg_user as given to
// lola_set_prefill_schedule, sms the device's SMs): one chain launch for the call or one
// per segment, and the intervals per segment (at most kMaxSegments segments per call).
// Automatic choice: one chain launch saves the chain the gap at every launch boundary
// (about 85 us on a B200), but holds its SMs for the whole call. Where the chain takes
// more than a third of the SMs, the attention beside it falls behind, and one launch per
// segment does better: between two chain launches the chain's SMs take waiting attention
// work, and the attention stays close behind the chain. Measured on a B200 (per call):
// 32 streams on 64 SMs, 256 intervals: 11.96 ms per segment vs 12.40 ms one launch;
// 8 streams on 40 SMs: 512 intervals 22.63 vs 23.19 ms, 64 intervals 1.17 vs 1.26 ms
// in favour of one launch. Segments of 16 intervals measured best in both forms; a
// shorter call (m intervals) keeps at least four segments of at least 8 intervals
// (32-interval calls: 18.75 ms per 16384 tokens in segments of 8, 19.06 in segments of 16).
void plan_schedule(const Dims &dm, int mode, int seg_user, int sms, int m, bool *one_chain, int *len)
{
    if (mode == LOLA_SCHEDULE_AUTO)
        mode = 3 * lola::chain_tc_prefill_ctas(dm) > sms ? LOLA_SCHEDULE_SEGMENTS : LOLA_SCHEDULE_ONE_CHAIN;
    int l = seg_user;
    if (l <= 0) {
        l = mode == LOLA_SCHEDULE_ONE_CHAIN ? std::max(16, dm.mmax / 32) : std::max(16, dm.mmax / 16);
        l = std::min(l, std::max(8, (m + 3) / 4));
    }
    *len = std::max(l, (dm.mmax + lola::kMaxSegments - 1) / lola::kMaxSegments);
    *one_chain = mode == LOLA_SCHEDULE_ONE_CHAIN;
}

}  // namespace

extern "C" {

const char *lola_status_string(lola_status s)
{
    switch (s) {
    case LOLA_OK: return "ok";
    case LOLA_ERR_INVALID_ARG: return "invalid argument";
    case LOLA_ERR_SHAPE: return "bad shape (n_tokens must be a positive multiple of chunk)";
    case LOLA_ERR_DTYPE: return "unsupported dtype";
    case LOLA_ERR_STATE: return "call not allowed at the state's position";
    case LOLA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case LOLA_ERR_CUDA: return "CUDA error";
    case LOLA_ERR_TIMEOUT: return "device wait timed out";
    case LOLA_ERR_DEVICE: return "device-side check failed";
    }
    return "unknown status";
}

lola_status lola_state_bytes(const lola_config *cfg, size_t *device_bytes)
{
    if (!device_bytes) return LOLA_ERR_INVALID_ARG;
    Dims dm;
    const lola_status r = derive_dims(cfg, &dm);
    if (r != LOLA_OK) return r;
    *device_bytes = layout(dm, nullptr, nullptr, nullptr);
    return LOLA_OK;
}

lola_status lola_state_stream_bytes(const lola_config *cfg, size_t *bytes)
{
    if (!bytes) return LOLA_ERR_INVALID_ARG;
    Dims dm;
    const lola_status r = derive_dims(cfg, &dm);
    if (r != LOLA_OK) return r;
    const size_t e = elem_bytes(dm);
    *bytes = (size_t)dm.D * dm.d * 4 + (size_t)dm.D * 4 + 2 * (size_t)dm.lam * dm.d * e +
             (size_t)dm.lam * 4 + 2 * (size_t)dm.R * dm.d * e + dm.Lmax;
    return LOLA_OK;
}

lola_status lola_init_state(const lola_config *cfg, const void *W, void *workspace,
                            size_t workspace_bytes, void *cuda_stream, lola_state **out)
{
    if (!cfg || !W || !workspace || !out) return LOLA_ERR_INVALID_ARG;
    Dims dm;
    lola_status r = derive_dims(cfg, &dm);
    if (r != LOLA_OK) return r;
    if (((uintptr_t)workspace & (kAlign - 1)) != 0) return LOLA_ERR_WORKSPACE;
    const size_t need = layout(dm, nullptr, nullptr, nullptr);
    if (workspace_bytes < need) return LOLA_ERR_WORKSPACE;
    lola_state *st = new (std::nothrow) lola_state();
    if (!st) return LOLA_ERR_INVALID_ARG;
    st->cfg = *cfg;
    st->dm = dm;
    st->ws = workspace;
    st->ws_bytes = workspace_bytes;
    layout(dm, (char *)workspace, &st->S, &st->P);
    reset_host(st);
    st->timing = false;
    st->overlap = false;
    st->sms = 0;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&st->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            cudaGetLastError();
    }
    st->sched_mode = LOLA_SCHEDULE_AUTO;
    st->seg_user = 0;
    st->chain_stream = nullptr;
    st->attn_stream = nullptr;
    st->seg_wait = wait_value_fn() != nullptr;
    for (int i = 0; i < lola::kMaxSegments; ++i) st->seg_expect[i] = 0;
    st->h2d_stream = st->d2h_stream = nullptr;
    if (segmented_prefill(dm)) {
        int lo = 0, hi = 0;
        bool okc = cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess &&
                   cudaStreamCreateWithPriority(&st->chain_stream, cudaStreamNonBlocking, hi) == cudaSuccess &&
                   cudaStreamCreateWithPriority(&st->attn_stream, cudaStreamNonBlocking, lo) == cudaSuccess &&
                   cudaEventCreateWithFlags(&st->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&st->ev_attn, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; okc && i < lola_state::kMaxSeg; ++i)
            okc = cudaEventCreateWithFlags(&st->ev_seg[i], cudaEventDisableTiming) == cudaSuccess;
        if (!okc) {
            cudaGetLastError();
            if (st->chain_stream != nullptr) cudaStreamDestroy(st->chain_stream);
            if (st->attn_stream != nullptr) cudaStreamDestroy(st->attn_stream);
            delete st;
            return LOLA_ERR_CUDA;
        }
        st->overlap = true;
    }
    const unsigned long long rk = (unsigned long long)dm.ns * (dm.lam + dm.R + dm.Nmax);
    const unsigned long long rv = (unsigned long long)dm.ns * (dm.lam + dm.R);
    if (dm.tc_chain && (!lola::make_row_map(&st->phik_map, st->P.phiK, rk, dm.D, 1) ||
                        !lola::make_row_map(&st->phik_box, st->P.phiK, rk, dm.D, 128) ||
                        !lola::make_row_map(&st->phiv_map, st->S.phiV, rv, dm.D, 1) ||
                        !lola::make_row_map(&st->phiv_box, st->S.phiV, rv, dm.D, 128))) {
        fprintf(stderr, "lola: cuTensorMapEncodeTiled failed (phi row maps)\n");
        cudaGetLastError();
        if (st->chain_stream != nullptr) cudaStreamDestroy(st->chain_stream);
        if (st->attn_stream != nullptr) cudaStreamDestroy(st->attn_stream);
        delete st;
        return LOLA_ERR_CUDA;
    }
    if (dm.dec_tma && !lola::make_decode_maps(dm, st->S, &st->maps)) {
        fprintf(stderr, "lola: cuTensorMapEncodeTiled failed\n");
        cudaGetLastError();
        if (st->chain_stream != nullptr) cudaStreamDestroy(st->chain_stream);
        if (st->attn_stream != nullptr) cudaStreamDestroy(st->attn_stream);
        delete st;
        return LOLA_ERR_CUDA;
    }
    lola::launch_init_state(dm, st->S, W, (cudaStream_t)cuda_stream);
    counted(1);
    r = check_launch();
    if (r != LOLA_OK) {
        delete st;
        return r;
    }
    *out = st;
    return LOLA_OK;
}

lola_status lola_reset_state(lola_state *st, void *cuda_stream)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    reset_host(st);
    {
        PhaseScope ps(st, PH_RESET, (cudaStream_t)cuda_stream);
        lola::launch_init_state(st->dm, st->S, nullptr, (cudaStream_t)cuda_stream);
        counted(1);
    }
    return check_launch();
}

int64_t lola_position(const lola_state *st) { return st ? st->pos : -1; }

lola_status lola_prefill_chunk(lola_state *st, const void *q, const void *k, const void *v,
                               int64_t n_tokens, void *out, void *cuda_stream)
{
    if (!st || !q || !k || !v || !out) return LOLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return LOLA_ERR_INVALID_ARG;
    const Dims &dm = st->dm;
    if (n_tokens <= 0 || n_tokens % dm.C != 0) return LOLA_ERR_SHAPE;
    if (n_tokens > dm.Nmax) return LOLA_ERR_WORKSPACE;
    if (st->pos != st->interval_end) return LOLA_ERR_STATE;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    const int n = (int)n_tokens;
    const int m = n / dm.C;
    const long long pos0 = st->pos;

    {
        // phi of the keys (cache slots, ring, call tokens); phi of the queries is
        // computed inside the tensor-core attention kernel
        PhaseScope ps(st, PH_PHI, stream);
        if (dm.dtype == LOLA_BF16) {
            lola::launch_phi_kv_tc(dm, st->S, k, pos0, n, dm.lam + dm.R + dm.Nmax, st->P.phiK, st->nS,
                                   stream);
            counted(1);
            if (!dm.tc_attn) {
                lola::launch_phi_q_tc(dm, st->S, q, (long long)dm.B * n * dm.Hq, st->P.phiQ, stream);
                counted(1);
            }
        } else {
            lola::launch_phi_kv(dm, st->S, k, pos0, n, dm.lam + dm.R + dm.Nmax, 0, st->P.phiK, st->nS,
                                stream);
            lola::launch_phi_q(dm, st->S.W, q, (long long)dm.B * n * dm.Hq, st->P.phiQ, stream);
            counted(2);
        }
    }
    if (check_launch() != LOLA_OK) return LOLA_ERR_CUDA;

    // The call's intervals run in segments. The chain (sequential per stream, a few SMs)
    // runs on the library's high-priority stream; the attention of a segment follows once
    // the chain has finished that segment, on the caller's stream or the second attention
    // stream, so it overlaps the chain of the next segments on the other SMs.
    bool one_chain = false;
    int seg = m;
    if (st->overlap) plan_schedule(dm, st->sched_mode, st->seg_user, st->sms, m, &one_chain, &seg);
    const int nseg = (m + seg - 1) / seg;
    const bool fork = nseg > 1 && st->chain_stream != nullptr;
    lola::AttnMaps amaps;
    if (dm.attn_ws) {
        lola::AttnArgs ma{};
        ma.n_call = n;
        ma.q = q;
        ma.kin = k;
        ma.vin = v;
        if (!lola::make_attn_maps(dm, ma, st->P.phiK, &amaps)) {
            fprintf(stderr, "lola: cuTensorMapEncodeTiled failed (prefill attention maps)\n");
            return LOLA_ERR_CUDA;
        }
    }
    cudaStream_t cs = fork ? st->chain_stream : stream;
    const bool two = fork && st->attn_stream != nullptr;
    if (fork) {
        cudaEventRecord(st->ev_fork, stream);
        cudaStreamWaitEvent(cs, st->ev_fork, 0);
        if (two) cudaStreamWaitEvent(st->attn_stream, st->ev_fork, 0);
    }
    // One chain launch for the whole call (where the schedule asks for it and the driver has
    // stream memory operations): the chain counts finished segments in device memory and the
    // attention of segment s waits for its count. Otherwise one chain launch per segment,
    // the attention gated by an event (plan_schedule weighs the two).
    const bool one = fork && one_chain && dm.tc_chain && st->seg_wait && nseg <= lola::kMaxSegments;
    for (int sg = 0; sg < nseg; ++sg) {
        const int ci0 = sg * seg;
        const int ms = m - ci0 < seg ? m - ci0 : seg;
        if (!one || sg == 0) {
            lola::ChainArgs ca{};
            ca.mode = 0;
            ca.pos0 = pos0 + (long long)ci0 * dm.C;
            ca.n_int = one ? m : ms;
            ca.ilen = dm.C;
            ca.call_start = pos0;
            ca.n_call = n;
            ca.kin = k;
            ca.vin = v;
            ca.nS0 = st->nS;
            ca.pend_lo = st->pend_lo;
            ca.pend_n = st->pend_n;
            ca.iglob0 = st->n_int;
            ca.phi = st->P.phiK;
            ca.nvrows = dm.lam + dm.R + dm.Nmax;
            ca.qin = q;
            ca.q_start = pos0;
            ca.q_n = n;
            ca.sel_log = st->sel_log;
            ca.sel_cap = st->sel_cap;
            ca.ovr = st->ovr;
            ca.ovr_n = st->ovr_n;
            ca.score_sre = st->score_sre;
            ca.score_tok = st->score_tok;
            ca.score_cap = st->score_cap;
            ca.inject_ns = take_injection(st, 1);
            ca.ci0 = ci0;
            ca.cont = sg > 0 ? 1 : 0;
            if (one) {
                ca.seg_done = st->S.seg_done;
                ca.seg_len = seg;
            }
            {
                PhaseScope ps(st, PH_CHAIN, cs);
                ca.snap_f32 = dm.tc_attn ? 0 : 1;
                if (dm.tc_chain) lola::launch_chain_tc(dm, st->S, &st->P, ca, st->phik_map, st->phik_box, cs);
                else lola::launch_chain(dm, st->S, &st->P, ca, cs);
                counted(1);
            }
            if (check_launch() != LOLA_OK) return LOLA_ERR_CUDA;
            if (one) {
                // the launched chain counts every segment of the call (also when it gives up),
                // so every target moves now, whatever happens to the attention launches below
                for (int s2 = 0; s2 < nseg; ++s2) st->seg_expect[s2] += (uint32_t)dm.ns;
            }
            if (fork) cudaEventRecord(st->ev_seg[sg], cs);
        }
        // the attention of this segment: on the caller's stream, or (odd segments) on the
        // second attention stream, after the segment's chain
        cudaStream_t as = (two && (sg & 1)) ? st->attn_stream : stream;
        if (one) {
            // every stream's chain has counted this segment (the count runs across calls)
            const uint32_t target = st->seg_expect[sg];
            if (wait_value_fn()((CUstream)as, (CUdeviceptr)(st->S.seg_done + sg), target, CU_STREAM_WAIT_VALUE_GEQ) !=
                CUDA_SUCCESS)
                cudaStreamWaitEvent(as, st->ev_seg[0], 0);   // the whole chain, then
        } else if (fork) {
            cudaStreamWaitEvent(as, st->ev_seg[sg], 0);
        }
        for (int ci = 0; ci < ms; ++ci) advance_interval(st, pos0 + (long long)(ci0 + ci) * dm.C, dm.C);

        lola::AttnArgs aa{};
        aa.pos0 = pos0;
        aa.m = ms;
        aa.ci0 = ci0;
        aa.n_call = n;
        aa.q = q;
        aa.kin = k;
        aa.vin = v;
        aa.out = out;
        {
            PhaseScope ps(st, PH_ATTN, as);
            if (dm.attn_ws) lola::launch_attn_ws(dm, st->S, st->P, aa, amaps, as);
            else if (dm.tc_attn) lola::launch_attn_tc(dm, st->S, st->P, aa, as);
            else lola::launch_attn_prefill(dm, st->S, st->P, aa, as);
            counted(1);
        }
        if (check_launch() != LOLA_OK) return LOLA_ERR_CUDA;
    }
    if (two) {
        // the caller's stream joins the second attention stream before the finalisation
        cudaEventRecord(st->ev_attn, st->attn_stream);
        cudaStreamWaitEvent(stream, st->ev_attn, 0);
    }
    if (one) cudaStreamWaitEvent(stream, st->ev_seg[0], 0);   // and the chain

    {
        PhaseScope ps(st, PH_FINAL, stream);
        lola::launch_finalize_prefill(dm, st->S, st->P, k, v, pos0, n, st->nS, stream);
        counted(2);
    }
    st->pos = pos0 + n;
    st->interval_end = st->pos;
    st->phiV_valid = false;   // cache slots and ring rows changed outside the decode path
    return check_launch();
}

lola_status lola_prefill_host_staging_bytes(const lola_config *cfg, int64_t piece_tokens, size_t *bytes)
{
    if (!bytes) return LOLA_ERR_INVALID_ARG;
    Dims dm;
    const lola_status r = derive_dims(cfg, &dm);
    if (r != LOLA_OK) return r;
    if (piece_tokens <= 0 || piece_tokens % dm.C != 0) return LOLA_ERR_SHAPE;
    if (piece_tokens > dm.Nmax) return LOLA_ERR_WORKSPACE;
    *bytes = 2 * host_slot(dm, piece_tokens).total;
    return LOLA_OK;
}

lola_status lola_prefill_host(lola_state *st, const void *q, const void *k, const void *v, int64_t n_tokens,
                              void *out, void *staging, size_t staging_bytes, int64_t piece_tokens,
                              void *cuda_stream)
{
    if (!st || !q || !k || !v || !out || !staging) return LOLA_ERR_INVALID_ARG;
    const Dims &dm = st->dm;
    if (n_tokens <= 0 || n_tokens % dm.C != 0 || piece_tokens <= 0 || piece_tokens % dm.C != 0)
        return LOLA_ERR_SHAPE;
    if (piece_tokens > dm.Nmax) return LOLA_ERR_WORKSPACE;
    if (((uintptr_t)staging & (kAlign - 1)) != 0) return LOLA_ERR_INVALID_ARG;
    const HostSlot hs = host_slot(dm, piece_tokens);
    if (staging_bytes < 2 * hs.total) return LOLA_ERR_WORKSPACE;
    if (st->pos != st->interval_end) return LOLA_ERR_STATE;
    if (!make_host_streams(st)) return LOLA_ERR_CUDA;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    const size_t e = elem_bytes(dm);
    const size_t qrow = (size_t)dm.Hq * dm.d * e, kvrow = (size_t)dm.Hkv * dm.d * e;   // bytes per token
    // the copy streams start after the caller's earlier work (which may still use the staging)
    cudaEventRecord(st->ev_host, stream);
    cudaStreamWaitEvent(st->h2d_stream, st->ev_host, 0);
    cudaStreamWaitEvent(st->d2h_stream, st->ev_host, 0);
    // the caller's stream passes this call once both copy streams are done (also after an
    // error, so that no copy into the caller's buffers outlives what the stream says)
    auto join = [&]() {
        cudaEventRecord(st->ev_host, st->h2d_stream);
        cudaStreamWaitEvent(stream, st->ev_host, 0);
        cudaEventRecord(st->ev_host, st->d2h_stream);
        cudaStreamWaitEvent(stream, st->ev_host, 0);
    };
    int i = 0;
    for (int64_t t0 = 0; t0 < n_tokens; t0 += piece_tokens, ++i) {
        const int64_t len = n_tokens - t0 < piece_tokens ? n_tokens - t0 : piece_tokens;
        const int slot = i & 1;
        char *qd = (char *)staging + (size_t)slot * hs.total;
        char *kd = qd + align_up(hs.q), *vd = kd + align_up(hs.kv), *od = vd + align_up(hs.kv);
        // inputs of this piece (rows t0 .. t0 + len of every sequence) into the slot, once the
        // compute of the piece two back has read it
        if (i >= 2) cudaStreamWaitEvent(st->h2d_stream, st->ev_comp[slot], 0);
        cudaMemcpy2DAsync(qd, (size_t)len * qrow, (const char *)q + (size_t)t0 * qrow, (size_t)n_tokens * qrow,
                          (size_t)len * qrow, (size_t)dm.B, cudaMemcpyHostToDevice, st->h2d_stream);
        cudaMemcpy2DAsync(kd, (size_t)len * kvrow, (const char *)k + (size_t)t0 * kvrow, (size_t)n_tokens * kvrow,
                          (size_t)len * kvrow, (size_t)dm.B, cudaMemcpyHostToDevice, st->h2d_stream);
        cudaMemcpy2DAsync(vd, (size_t)len * kvrow, (const char *)v + (size_t)t0 * kvrow, (size_t)n_tokens * kvrow,
                          (size_t)len * kvrow, (size_t)dm.B, cudaMemcpyHostToDevice, st->h2d_stream);
        cudaEventRecord(st->ev_h2d[slot], st->h2d_stream);
        // the piece: its inputs have landed and the slot's outputs of two pieces back are out
        cudaStreamWaitEvent(stream, st->ev_h2d[slot], 0);
        if (i >= 2) cudaStreamWaitEvent(stream, st->ev_d2h[slot], 0);
        const lola_status r = lola_prefill_chunk(st, qd, kd, vd, len, od, stream);
        if (r != LOLA_OK) {
            join();
            return r;
        }
        cudaEventRecord(st->ev_comp[slot], stream);
        // its outputs back to the host rows
        cudaStreamWaitEvent(st->d2h_stream, st->ev_comp[slot], 0);
        cudaMemcpy2DAsync((char *)out + (size_t)t0 * qrow, (size_t)n_tokens * qrow, od, (size_t)len * qrow,
                          (size_t)len * qrow, (size_t)dm.B, cudaMemcpyDeviceToHost, st->d2h_stream);
        cudaEventRecord(st->ev_d2h[slot], st->d2h_stream);
    }
    join();
    return check_launch();
}

lola_status lola_decode_step(lola_state *st, const void *q, const void *k, const void *v,
                             void *out, void *cuda_stream)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    return decode_step_impl(st, q, k, v, out, cuda_stream, st->S.part, st->S.phiQd);
}

lola_status lola_get_cache_indices(const lola_state *st, int32_t *dev_idx, int32_t *dev_count,
                                   void *cuda_stream)
{
    if (!st || !dev_idx) return LOLA_ERR_INVALID_ARG;
    lola::launch_get_indices(st->dm, st->S, st->nS, dev_idx, dev_count, (cudaStream_t)cuda_stream);
    counted(1);
    return check_launch();
}

lola_status lola_set_selection_log(lola_state *st, int32_t *dev_buf, int64_t capacity)
{
    if (!st || capacity < 0) return LOLA_ERR_INVALID_ARG;
    st->sel_log = dev_buf;
    st->sel_cap = dev_buf ? capacity : 0;
    return LOLA_OK;
}

lola_status lola_set_selection_override(lola_state *st, const int32_t *dev_kept, int64_t n_intervals)
{
    if (!st || n_intervals < 0) return LOLA_ERR_INVALID_ARG;
    st->ovr = dev_kept;
    st->ovr_n = dev_kept ? n_intervals : 0;
    return LOLA_OK;
}

lola_status lola_set_fault_injection(lola_state *st, int32_t where, int64_t wait_limit_ns)
{
    if (!st || where < 0 || where > 2 || (where != 0 && (wait_limit_ns <= 0 || wait_limit_ns > 2000000000LL)))
        return LOLA_ERR_INVALID_ARG;
    if (where == 1 && !st->dm.tc_chain) return LOLA_ERR_INVALID_ARG;   // the hook sits in the tensor-core chain
    if (where == 2 && st->dm.dtype != LOLA_BF16) return LOLA_ERR_INVALID_ARG;
    st->inject_where = where;
    st->inject_ns = where ? (unsigned long long)wait_limit_ns : 0;
    return LOLA_OK;
}

lola_status lola_set_score_log(lola_state *st, float *dev_sre, int32_t *dev_tok, int64_t capacity)
{
    if (!st || capacity < 0 || ((dev_sre == nullptr) != (dev_tok == nullptr))) return LOLA_ERR_INVALID_ARG;
    st->score_sre = dev_sre;
    st->score_tok = dev_tok;
    st->score_cap = dev_sre ? capacity : 0;
    return LOLA_OK;
}

lola_status lola_sync(lola_state *st, void *cuda_stream)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return check_launch();
    int err[4] = {0, 0, 0, 0};
    if (cudaMemcpy(err, st->S.err, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess)
        return check_launch();
    if (err[0] != 0) {
        // A kernel that gave up left its work unfinished, including the per-stream
        // counters by which the decode kernels find the last partial of a stream:
        // they restart from zero, and the caller resets the state (lola_reset_state)
        // before using it again.
        cudaMemset(st->S.err, 0, sizeof(err));
        cudaMemset(st->S.dec_cnt, 0, (size_t)st->dm.ns * sizeof(int));
        return (err[0] & lola::ERR_TIMEOUT) ? LOLA_ERR_TIMEOUT : LOLA_ERR_DEVICE;
    }
    return LOLA_OK;
}

lola_status lola_set_prefill_schedule(lola_state *st, int32_t mode, int32_t intervals_per_segment)
{
    if (!st || intervals_per_segment < 0) return LOLA_ERR_INVALID_ARG;
    if (mode != LOLA_SCHEDULE_AUTO && mode != LOLA_SCHEDULE_ONE_CHAIN && mode != LOLA_SCHEDULE_SEGMENTS)
        return LOLA_ERR_INVALID_ARG;
    st->sched_mode = mode;
    st->seg_user = intervals_per_segment;
    return LOLA_OK;
}

lola_status lola_prefill_plan(const lola_config *cfg, int32_t mode, int32_t intervals_per_segment, int32_t sms,
                              int64_t n_tokens, int32_t *mode_out, int32_t *len_out, int32_t *segments_out)
{
    if (!mode_out || !len_out || !segments_out || sms < 1 || intervals_per_segment < 0) return LOLA_ERR_INVALID_ARG;
    if (mode != LOLA_SCHEDULE_AUTO && mode != LOLA_SCHEDULE_ONE_CHAIN && mode != LOLA_SCHEDULE_SEGMENTS)
        return LOLA_ERR_INVALID_ARG;
    Dims dm;
    const lola_status r = derive_dims(cfg, &dm);
    if (r != LOLA_OK) return r;
    if (n_tokens <= 0 || n_tokens % dm.C != 0) return LOLA_ERR_SHAPE;
    if (n_tokens > dm.Nmax) return LOLA_ERR_WORKSPACE;
    const int m = (int)(n_tokens / dm.C);
    bool one = false;
    int len = m;
    if (segmented_prefill(dm)) plan_schedule(dm, mode, intervals_per_segment, sms, m, &one, &len);
    const int nseg = (m + len - 1) / len;
    *mode_out = one && nseg > 1 ? LOLA_SCHEDULE_ONE_CHAIN : LOLA_SCHEDULE_SEGMENTS;
    *len_out = nseg > 1 ? len : m;
    *segments_out = nseg;
    return LOLA_OK;
}

lola_status lola_set_timing(lola_state *st, int enable)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    st->timing = enable != 0;
    return LOLA_OK;
}

lola_status lola_timing_read(lola_state *st, double *ms, int64_t *n)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    lola_status r = LOLA_OK;
    for (auto &mk : st->marks) {
        float t = 0.f;
        if (cudaEventSynchronize(mk.b) != cudaSuccess || cudaEventElapsedTime(&t, mk.a, mk.b) != cudaSuccess)
            r = LOLA_ERR_CUDA;
        if (ms && mk.phase < 8) ms[mk.phase] += t;
        if (n && mk.phase < 8) n[mk.phase] += 1;
        st->pool.push_back(mk.a);
        st->pool.push_back(mk.b);
    }
    st->marks.clear();
    if (r != LOLA_OK) check_launch();
    return r;
}

int64_t lola_launch_count(void) { return g_launches.load(); }

lola_status lola_free_state(lola_state *st)
{
    if (!st) return LOLA_OK;
    for (auto &mk : st->marks) {
        st->pool.push_back(mk.a);
        st->pool.push_back(mk.b);
    }
    for (cudaEvent_t e : st->pool) cudaEventDestroy(e);
    if (st->chain_stream != nullptr) {
        cudaStreamSynchronize(st->chain_stream);
        cudaStreamDestroy(st->chain_stream);
        cudaEventDestroy(st->ev_fork);
        for (int i = 0; i < lola_state::kMaxSeg; ++i) cudaEventDestroy(st->ev_seg[i]);
    }
    if (st->attn_stream != nullptr) {
        cudaStreamSynchronize(st->attn_stream);
        cudaStreamDestroy(st->attn_stream);
        cudaEventDestroy(st->ev_attn);
    }
    if (st->h2d_stream != nullptr) {
        cudaStreamSynchronize(st->h2d_stream);
        cudaStreamSynchronize(st->d2h_stream);
        cudaStreamDestroy(st->h2d_stream);
        cudaStreamDestroy(st->d2h_stream);
        for (int i = 0; i < 2; ++i) {
            cudaEventDestroy(st->ev_h2d[i]);
            cudaEventDestroy(st->ev_comp[i]);
            cudaEventDestroy(st->ev_d2h[i]);
        }
        cudaEventDestroy(st->ev_host);
    }
    delete st;
    return LOLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- decode step, library-owned scratch
//
// lola_decode_step_static runs the same decode step as lola_decode_step, but
// the per-step temporaries of the decode attention (the partial sums of the
// warps or CTAs that share a stream, and the query features) live in the
// fixed device array below
// instead of the caller's workspace. It exists for callers that cannot obtain
// device memory on demand: a host framework that owns all device memory and
// hands a plugin only its inputs, outputs and persistent state, or code that
// runs while a CUDA graph is being captured, where cudaMalloc is not allowed.
// The array is part of the library image, so every GPU that loads the library
// holds it until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
lola_status static_scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LOLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress((void **)&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) {
            fprintf(stderr, "lola: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
            return LOLA_ERR_CUDA;
        }
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return LOLA_OK;
}

}  // namespace

extern "C" lola_status lola_decode_step_static(lola_state *st, const void *q, const void *k,
                                               const void *v, void *out, void *cuda_stream)
{
    if (!st) return LOLA_ERR_INVALID_ARG;
    const Dims &dm = st->dm;
    const size_t part_bytes = align_up((size_t)dm.ns * dm.nsplit * dm.g * (2 * dm.d + 4) * 4);
    const size_t phiq_bytes = dm.dtype == LOLA_BF16 ? align_up((size_t)dm.B * dm.Hq * dm.D * 4) : 0;
    if (part_bytes + phiq_bytes > kStaticScratchBytes) return LOLA_ERR_WORKSPACE;
    void *base = nullptr;
    const lola_status sr = static_scratch_address(&base);
    if (sr != LOLA_OK) return sr;
    // Every partial and query feature is written before it is read within one
    // call, so nothing has to start at zero.
    return decode_step_impl(st, q, k, v, out, cuda_stream, (float *)base,
                            phiq_bytes ? (float *)((char *)base + part_bytes) : nullptr);
}
