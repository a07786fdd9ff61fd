// Alternative candidate scores for the sparse cache: the scoring methods LoLA's
// ablations compare the Self-Recall Error against (gist.science technical
// summary, "Belangrijkste bijdragen" and "Ablaties": the magnitude of attention
// weights, a softmax-approximation error) and the FIFO structure the
// "Inferentiestrategie" section mentions. This engine's readings, for the
// interval's first query q (token t0), summed over the g query heads of the
// stream's group:
//   kAttnWeight:   a_c = softmax over the candidates of q.k_c / sqrt(d);
//   kSoftmaxError: (a_c - b_c)^2, b_c = phi(q).phi(k_c) / sum over candidates;
//   kRecency:      the token index (the most recent pairs stay).
// The highest scores stay cached, as with the SRE.
#pragma once

#include "lola_internal.cuh"

namespace lola {

enum : int { kScoreSRE = 0, kAttnWeight = 1, kSoftmaxError = 2, kRecency = 3 };

// dot product of a row of T (16-byte aligned, n a multiple of 16 / sizeof(T)) with fp32 v
template <typename T> __device__ __forceinline__ float dot_row(const T *__restrict__ row, const float *v, int n)
{
    constexpr int VN = 16 / sizeof(T);
    float acc = 0.f;
    for (int e = 0; e < n; e += VN) {
        const uint4 r = *(const uint4 *)(row + e);
        const T *x = (const T *)&r;
#pragma unroll
        for (int i = 0; i < VN; ++i) acc = fmaf(to_f<T>(x[i]), v[e + i], acc);
    }
    return acc;
}

// Block-wide max (op 0) or sum (op 1) of one value per thread; red: >= 32 floats
// of shared memory. Every thread gets the result.
__device__ __forceinline__ float block_reduce(float x, int op, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, x, o);
        x = op == 0 ? fmaxf(x, y) : x + y;
    }
    __syncthreads();   // earlier readers of red are done
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = op == 0 ? -INFINITY : 0.f;
    for (int w = 0; w < nw; ++w) r = op == 0 ? fmaxf(r, red[w]) : r + red[w];
    return r;
}

// Scores of the nQ candidates (whole CTA; needs at least g warps). krow(c) / prow(c)
// return candidate c's key row (d elements) / phi row (D elements) in dtype T, tok(c)
// its token; qrow(h) the interval's first query of group head h (d elements). W is
// the fp32 feature-map matrix [d][D/2]. Shared scratch: qs [g*d], pq [g*D], lg [nQ],
// lu [nQ], red [32] (floats); score [nQ] receives the scores.
template <typename T, typename KRow, typename PRow, typename QRow, typename Tok>
__device__ void alt_scores(int kind, int nQ, KRow krow, PRow prow, QRow qrow, Tok tok, const float *__restrict__ W,
                           int g, int d, int D, float *score, float *qs, float *pq, float *lg, float *lu, float *red)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    if (kind == kRecency) {
        for (int c = tid; c < nQ; c += nt) score[c] = (float)tok(c);
        __syncthreads();
        return;
    }
    const int Dh = D / 2;
    for (int e = tid; e < g * d; e += nt) qs[e] = to_f<T>(qrow(e / d)[e % d]);
    for (int c = tid; c < nQ; c += nt) score[c] = 0.f;
    __syncthreads();
    if (kind == kSoftmaxError) {
        // phi(q_h) = [softmax(q_h W), softmax(-q_h W)]: z, then one warp per head
        for (int e = tid; e < g * Dh; e += nt) {
            const int h = e / Dh, j = e - h * Dh;
            float z = 0.f;
            for (int a = 0; a < d; ++a) z = fmaf(qs[h * d + a], W[(size_t)a * Dh + j], z);
            pq[h * D + j] = z;
        }
        __syncthreads();
        if (warp < g) {
            float *ph = pq + warp * D;
            float zmax = -INFINITY, zmin = INFINITY;
            for (int j = lane; j < Dh; j += 32) {
                zmax = fmaxf(zmax, ph[j]);
                zmin = fminf(zmin, ph[j]);
            }
            zmax = warp_max(zmax);
            zmin = warp_min(zmin);
            float sp = 0.f, sn = 0.f;
            for (int j = lane; j < Dh; j += 32) {
                sp += __expf(ph[j] - zmax);
                sn += __expf(zmin - ph[j]);
            }
            sp = warp_sum(sp);
            sn = warp_sum(sn);
            __syncwarp();
            for (int j = lane; j < Dh; j += 32) {
                const float z = ph[j];
                ph[j] = __expf(z - zmax) / sp;
                ph[Dh + j] = __expf(zmin - z) / sn;
            }
        }
        __syncthreads();
    }
    const float scale = rsqrtf((float)d);
    for (int h = 0; h < g; ++h) {
        float mx = -INFINITY, us = 0.f;
        for (int c = tid; c < nQ; c += nt) {
            const float l = dot_row<T>(krow(c), qs + h * d, d) * scale;
            lg[c] = l;
            mx = fmaxf(mx, l);
            if (kind == kSoftmaxError) {
                const float u = dot_row<T>(prow(c), pq + h * D, D);
                lu[c] = u;
                us += u;
            }
        }
        const float M = block_reduce(mx, 0, red);
        const float U = kind == kSoftmaxError ? block_reduce(us, 1, red) : 1.f;
        float zs = 0.f;
        for (int c = tid; c < nQ; c += nt) {
            const float e = __expf(lg[c] - M);
            lg[c] = e;
            zs += e;
        }
        const float rZ = 1.f / block_reduce(zs, 1, red);
        const float rU = U > 0.f ? 1.f / U : 0.f;
        for (int c = tid; c < nQ; c += nt) {
            const float a = lg[c] * rZ;
            if (kind == kAttnWeight) {
                score[c] += a;
            } else {
                const float e = a - lu[c] * rU;
                score[c] = fmaf(e, e, score[c]);
            }
        }
        __syncthreads();
    }
}

}  // namespace lola
