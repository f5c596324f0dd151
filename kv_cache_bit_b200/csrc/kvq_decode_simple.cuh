// kvq_decode_simple.cuh -- split-K decode attention over the packed cache,
// CUDA-core (FFMA) form.  One CTA per (sequence split, batch*kv-head) handles
// all G query heads of that kv head; the partial softmax states of the splits
// are merged by decode_combine_kernel.  Included once, by kvq_api.cu.
//
// With w_t = q_t (.) sigma_b (codes times the block's channel scales) the
// attention is computed without expanding the cache:
//   logit_t = scale * kappa_t * sum_c q'_c code_{t,c}  [+ scale s1_t (q . o_b)]
//   acc    += p_t nu_t code_t, multiplied by sigma^V_b once per block
// with q' = qt (.) sigma^K_b, where qt = H(s (.) q) under HADAMARD, else q:
//   nsep    kappa = nu = n (times 1/sqrt(d) under HADAMARD)
//   naive   kappa = nu = per-token scale, sigma = 1
//   NSN     kappa = s1 s2 (times sqrt(d) without HADAMARD), nu likewise,
//           plus beta_b = sum_{t in b} p_t s1_t times o^V_b
// The output is (s (.) H(acc) under HADAMARD, else acc) + acc_o, divided by
// the softmax sum; residual tokens enter acc_o at their fp16 values.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

constexpr int kGMax = 8;  // query heads per kv head handled by one CTA

struct DecodeArgs {
    const uint8_t* codes[2];
    const __half* tok[2];
    const __half* chan[2];
    const __half* off[2];
    const __half* resid[2];
    const __half* q;   // [B][H*G][D]
    float* out;        // [B][H*G][D]
    float* part;       // [B*H][nsplit][G][2 + 2D]: m, l, acc[D], acc_o[D]
    const int8_t* signs;
    int H, G, cap, nbq, rlen, nsplit, bps;
    long long work;    // tensor-core path: quantized blocks of all pairs
    long long nwarps;  // tensor-core path: warps of the persistent grid
    float scale, rsqd, sqd;
};

template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) decode_split_kernel(DecodeArgs a) {
    using L = RowLayout<D, BITS>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int G = a.G;
    const int nb_cap = a.cap / kT;
    const int ntk = tok_params(MODE);
    constexpr int OW = off_words<D, MODE>();

    __shared__ float s_qo[kGMax][D];   // queries, original domain
    __shared__ float s_qt[kGMax][D];   // queries, rotated domain (HADAMARD)
    __shared__ float s_qp[kGMax][D];   // q' of the current block
    __shared__ float s_lg[kGMax][kT];  // logits, then p * nu
    __shared__ float s_sigv[D], s_offv[D], s_offk[D];
    __shared__ float s_nu[kT], s_s1[kT];
    __shared__ uint32_t s_vw[kT][RowLayout<D, BITS>::kWords];  // V code rows of the current block
    __shared__ float s_m[kGMax], s_l[kGMax], s_corr[kGMax], s_beta[kGMax], s_qok[kGMax];

    const int b = bh / a.H, h = bh % a.H;
    for (int i = t; i < G * D; i += 128) {
        const int j = i / D, c = i % D;
        const float qv = __half2float(a.q[((size_t)b * a.H * G + (size_t)h * G + j) * D + c]);
        s_qo[j][c] = qv;
        s_qt[j][c] = qv;
    }
    if (t < kGMax) { s_m[t] = -INFINITY; s_l[t] = 0.0f; }
    __syncthreads();
    if constexpr (HAD) {
        if (t < G) {
            float r[D];
#pragma unroll
            for (int c = 0; c < D; ++c) r[c] = (a.signs != nullptr && a.signs[c] < 0) ? -s_qo[t][c] : s_qo[t][c];
            fwht_reg<D>(r);
#pragma unroll
            for (int c = 0; c < D; ++c) s_qt[t][c] = r[c];
        }
        __syncthreads();
    }

    float acc[kGMax], acco[kGMax];
#pragma unroll
    for (int j = 0; j < kGMax; ++j) { acc[j] = 0.0f; acco[j] = 0.0f; }

    const int blk_begin = split * a.bps;
    const int blk_end = min(a.nbq, blk_begin + a.bps);
    for (int blk = blk_begin; blk < blk_end; ++blk) {
        // 1. block parameters and q'
        const uint8_t* reck = nullptr;
        const uint8_t* recv = nullptr;
        if constexpr (MODE == kNsnDq) {
            reck = reinterpret_cast<const uint8_t*>(a.off[0] + ((size_t)bh * nb_cap + blk) * OW);
            recv = reinterpret_cast<const uint8_t*>(a.off[1] + ((size_t)bh * nb_cap + blk) * OW);
        }
        if (t < D) {
            const size_t bi = ((size_t)bh * nb_cap + blk) * D + t;
            const float sk = (MODE != kNaive) ? __half2float(a.chan[0][bi]) : 1.0f;
            s_sigv[t] = (MODE != kNaive) ? __half2float(a.chan[1][bi]) : 1.0f;
            if (MODE == kNsn) {
                s_offk[t] = __half2float(a.off[0][bi]);
                s_offv[t] = __half2float(a.off[1][bi]);
            }
            if (MODE == kNsnDq) {
                s_offk[t] = dq_o<D>(reck, t);
                s_offv[t] = dq_o<D>(recv, t);
            }
            for (int j = 0; j < G; ++j) s_qp[j][t] = s_qt[j][t] * sk;
        }
        __syncthreads();
        if constexpr (is_nsn(MODE)) {
            for (int j = warp; j < G; j += 4) {
                float s = 0.0f;
                for (int c = lane; c < D; c += 32) s += s_qo[j][c] * s_offk[c];
#pragma unroll
                for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) s_qok[j] = s;
            }
            __syncthreads();
        }
        // 2. logits, one token per thread
        {
            const size_t ti = (size_t)bh * a.cap + (size_t)blk * kT + t;
            uint32_t w[L::kWords];
            load_words<L::kWords>(a.codes[0] + ti * L::kBytes, w);
            float sj[kGMax];
#pragma unroll
            for (int j = 0; j < kGMax; ++j) sj[j] = 0.0f;
#pragma unroll
            for (int c = 0; c < D; ++c) {
                const float q = (float)((int)code_at<D, BITS>(w, c) - L::kOff);
#pragma unroll
                for (int j = 0; j < kGMax; ++j)
                    if (j < G) sj[j] += s_qp[j][c] * q;
            }
            const __half* tp = a.tok[0] + ti * ntk;
            const __half* tv = a.tok[1] + ti * ntk;
            float kap, nu, s1k = 0.0f, s1v = 0.0f;
            if constexpr (MODE == kNsn) {
                s1k = __half2float(tp[0]);
                kap = s1k * __half2float(tp[1]) * (HAD ? 1.0f : a.sqd);
                s1v = __half2float(tv[0]);
                nu = s1v * __half2float(tv[1]) * (HAD ? 1.0f : a.sqd);
            } else if constexpr (MODE == kNsnDq) {
                s1k = dq_s1<D>(reck, t);
                kap = s1k * __half2float(tp[0]) * (HAD ? 1.0f : a.sqd);
                s1v = dq_s1<D>(recv, t);
                nu = s1v * __half2float(tv[0]) * (HAD ? 1.0f : a.sqd);
            } else {
                kap = __half2float(tp[0]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                nu = __half2float(tv[0]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
            }
            for (int j = 0; j < G; ++j) {
                float lg = kap * sj[j];
                if (is_nsn(MODE)) lg += s1k * s_qok[j];
                s_lg[j][t] = a.scale * lg;
            }
            s_nu[t] = nu;
            s_s1[t] = s1v;
        }
        __syncthreads();
        // 3. online softmax per head (one warp per head)
        for (int j = warp; j < G; j += 4) {
            float m = -INFINITY;
            for (int i = lane; i < kT; i += 32) m = fmaxf(m, s_lg[j][i]);
#pragma unroll
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float mold = s_m[j];
            const float mnew = fmaxf(mold, m);
            float ps = 0.0f, bs = 0.0f;
            for (int i = lane; i < kT; i += 32) {
                const float p = __expf(s_lg[j][i] - mnew);
                ps += p;
                bs += p * s_s1[i];
                s_lg[j][i] = p * s_nu[i];
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                ps += __shfl_xor_sync(0xffffffffu, ps, o);
                bs += __shfl_xor_sync(0xffffffffu, bs, o);
            }
            if (lane == 0) {
                const float corr = __expf(mold - mnew);
                s_corr[j] = corr;
                s_l[j] = s_l[j] * corr + ps;
                s_m[j] = mnew;
                s_beta[j] = bs;
            }
        }
        __syncthreads();
        // 4. V accumulation, one channel per thread, from the block's V code
        //    rows staged in shared memory (thread i copies row i)
        {
            const uint8_t* vrow = a.codes[1] + ((size_t)bh * a.cap + (size_t)blk * kT + t) * L::kBytes;
            uint32_t w[L::kWords];
            load_words<L::kWords>(vrow, w);
#pragma unroll
            for (int k = 0; k < L::kWords; ++k) s_vw[t][k] = w[k];
        }
        __syncthreads();
        if (t < D) {
            float aj[kGMax];
#pragma unroll
            for (int j = 0; j < kGMax; ++j) aj[j] = 0.0f;
#pragma unroll 4
            for (int i = 0; i < kT; ++i) {
                const float q = (float)((int)code_at<D, BITS>(s_vw[i], t) - L::kOff);
#pragma unroll
                for (int j = 0; j < kGMax; ++j)
                    if (j < G) aj[j] += s_lg[j][i] * q;
            }
#pragma unroll
            for (int j = 0; j < kGMax; ++j) {
                if (j < G) {
                    acc[j] = acc[j] * s_corr[j] + s_sigv[t] * aj[j];
                    acco[j] = acco[j] * s_corr[j] + (is_nsn(MODE) ? s_beta[j] * s_offv[t] : 0.0f);
                }
            }
        }
        __syncthreads();
    }

    // residual tokens (fp16), last split only
    if (split == a.nsplit - 1 && a.rlen > 0) {
        const __half* rk = a.resid[0] + (size_t)bh * kT * D;
        const __half* rv = a.resid[1] + (size_t)bh * kT * D;
        if (t < a.rlen) {
            for (int j = 0; j < G; ++j) {
                float s = 0.0f;
                for (int c = 0; c < D; ++c) s += s_qo[j][c] * __half2float(rk[(size_t)t * D + c]);
                s_lg[j][t] = a.scale * s;
            }
        } else {
            for (int j = 0; j < G; ++j) s_lg[j][t] = -INFINITY;
        }
        __syncthreads();
        for (int j = warp; j < G; j += 4) {
            float m = -INFINITY;
            for (int i = lane; i < kT; i += 32) m = fmaxf(m, s_lg[j][i]);
#pragma unroll
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float mold = s_m[j];
            const float mnew = fmaxf(mold, m);
            float ps = 0.0f;
            for (int i = lane; i < kT; i += 32) {
                const float p = (i < a.rlen) ? __expf(s_lg[j][i] - mnew) : 0.0f;
                ps += p;
                s_lg[j][i] = p;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            if (lane == 0) {
                const float corr = __expf(mold - mnew);
                s_corr[j] = corr;
                s_l[j] = s_l[j] * corr + ps;
                s_m[j] = mnew;
            }
        }
        __syncthreads();
        if (t < D) {
            float aj[kGMax];
#pragma unroll
            for (int j = 0; j < kGMax; ++j) aj[j] = 0.0f;
            for (int i = 0; i < a.rlen; ++i) {
                const float x = __half2float(rv[(size_t)i * D + t]);
#pragma unroll
                for (int j = 0; j < kGMax; ++j)
                    if (j < G) aj[j] += s_lg[j][i] * x;
            }
#pragma unroll
            for (int j = 0; j < kGMax; ++j) {
                if (j < G) {
                    acc[j] = acc[j] * s_corr[j];
                    acco[j] = acco[j] * s_corr[j] + aj[j];
                }
            }
        }
        __syncthreads();
    }

    float* pp = a.part + ((size_t)bh * a.nsplit + split) * G * (2 + 2 * D);
    for (int j = 0; j < G; ++j) {
        float* pj = pp + (size_t)j * (2 + 2 * D);
        if (t == 0) { pj[0] = s_m[j]; pj[1] = s_l[j]; }
        if (t < D) {
            float aa = 0.0f, ao = 0.0f;
#pragma unroll
            for (int jj = 0; jj < kGMax; ++jj)
                if (jj == j) { aa = acc[jj]; ao = acco[jj]; }
            pj[2 + t] = aa;
            pj[2 + D + t] = ao;
        }
    }
}

// Merge the splits of one (batch, kv head): log-sum-exp weights, inverse
// rotation of the code term, division by the softmax sum.
template <int D, bool HAD>
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeArgs a) {
    const int t = threadIdx.x, bh = blockIdx.x;
    const int G = a.G;
    const int b = bh / a.H, h = bh % a.H;
    __shared__ float s_a[kGMax][D];
    __shared__ float s_w[64];
    const float* pp = a.part + (size_t)bh * a.nsplit * G * (2 + 2 * D);
    float ao[kGMax], inv_l[kGMax];
    for (int j = 0; j < G; ++j) {
        float M = -INFINITY;
        for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, pp[((size_t)s * G + j) * (2 + 2 * D)]);
        float Lsum = 0.0f, A = 0.0f, AO = 0.0f;
        for (int s = 0; s < a.nsplit; ++s) {
            const float* ps = pp + ((size_t)s * G + j) * (2 + 2 * D);
            const float wgt = (ps[0] == -INFINITY) ? 0.0f : __expf(ps[0] - M);
            Lsum += wgt * ps[1];
            if (t < D) {
                A += wgt * ps[2 + t];
                AO += wgt * ps[2 + D + t];
            }
        }
        if (t < D) s_a[j][t] = A;
        ao[j < kGMax ? j : 0] = AO;
        inv_l[j < kGMax ? j : 0] = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
    }
    (void)s_w;
    __syncthreads();
    if constexpr (HAD) {
        if (t < G) {
            float r[D];
#pragma unroll
            for (int c = 0; c < D; ++c) r[c] = s_a[t][c];
            fwht_reg<D>(r);
#pragma unroll
            for (int c = 0; c < D; ++c) s_a[t][c] = (a.signs != nullptr && a.signs[c] < 0) ? -r[c] : r[c];
        }
        __syncthreads();
    }
    if (t < D) {
        for (int j = 0; j < G; ++j)
            a.out[((size_t)b * a.H * G + (size_t)h * G + j) * D + t] = (s_a[j][t] + ao[j]) * inv_l[j];
    }
}

}  // namespace kvq
