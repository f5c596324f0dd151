// kvq_decode_mma.cuh -- decode attention over the packed cache on the tensor
// cores (head dim 128).  Included once, by kvq_api.cu.
//
// Work: grid (split, batch*kv-head); a CTA of kNW warps covers a contiguous
// range of 128-token blocks of one (batch, kv head); warp w takes blocks
// w, w + kNW, ... of the range, each warp an independent online-softmax
// partial.  Each warp owns a ring of kRing shared-memory slots; a slot holds
// one tensor's half of a block (packed codes, per-token parameters, channel
// scales and NSN means), brought in by 1-D bulk copies (no multicast) that
// complete on the slot's mbarrier.  The order of slots is K(b0), V(b0),
// K(b1), V(b1), ...
//
// Per block (all G query heads of the kv head at once, G <= 8):
//   scores  S[tok][col] = sum_c code[tok][c] * q'[c][col] with
//           mma.m16n8k16 (A = codes, unpacked from nibbles straight into the
//           fragment registers; B = q' = qt (.) sigma^K scaled by a power of
//           two and split into fp16 hi + lo columns, so the fp32 operand
//           keeps ~22 bits; codes are exact in fp16).
//   softmax logits in the log2 domain, online max/sum per head.
//   values  Acc[c][col] += sum_tok code^V[tok][c] * P'[tok][col] with
//           mma.m16n8k16 (A = V codes transposed, two token rows interleaved
//           by byte permutes; B = P' = p * nu split into hi + lo, moved from
//           the score accumulator layout into the B layout with movmatrix),
//           then scaled by sigma^V of the block into fp32 accumulators.
// The channel and token orders inside a fragment are permutations chosen so
// that every unpack step is a few byte/bit operations; A and B always use the
// same permutation, and the sums are order-free up to rounding.
#pragma once

#include "kvq_decode_simple.cuh"
#include "kvq_device.cuh"

namespace kvq {

constexpr int kNW = 4;    // consumer warps per CTA
constexpr int kRing = 2;  // slots per warp

// ---------------------------------------------------------------- small PTX helpers

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t m, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(m), "r"(c));  // (a & m) | c
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t h2_sub(uint32_t x, uint32_t y) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
    return r;
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t x, uint32_t y, uint32_t z) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(y), "r"(z));
    return r;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t r;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

// D += A * B, m16n8k16, fp16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 2^k for integer k in [-126, 127].
__device__ __forceinline__ float pow2i(int k) {
    k = max(-126, min(127, k));
    return __uint_as_float(uint32_t(k + 127) << 23);
}

// ceil(log2(x)) for x > 0 normal.
__device__ __forceinline__ int ceil_log2(float x) {
    const uint32_t b = __float_as_uint(x);
    const int e = int((b >> 23) & 0xFF) - 127;
    return (b & 0x7FFFFF) ? e + 1 : e;
}

constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 1024.0, 1024.0

__device__ __forceinline__ uint32_t h2c(float v) { return pack_h2(v, v); }

// ---------------------------------------------------------------- code unpacking

// K side.  Thread slot t of a quad owns channels [32t, 32t + 32) of a token
// row and turns them into 16 fp16x2 pairs; pair p holds the codes of
// channels (kc_a(p), kc_b(p)) relative to 32t.
template <int BITS>
struct KUnpack;

template <>
struct KUnpack<4> {
    static constexpr int kSliceBytes = 16;
    __device__ static int ca(int p) { return 8 * (p >> 2) + (p & 3); }
    __device__ static int cb(int p) { return ca(p) + 4; }
    // row points at the row's first byte; returns pairs of codes (q = e - 8)
    __device__ static void run(const uint8_t* row, int t, uint32_t (&pr)[16]) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * t);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        const uint32_t sub = h2c(1032.0f), s16 = h2c(1.0f / 16.0f), o16 = h2c(-72.0f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t W = w[i], W8 = w[i] >> 8;
            pr[4 * i + 0] = h2_sub(lop_and_or(W, 0x000F000Fu, kMagic), sub);
            pr[4 * i + 1] = h2_fma(lop_and_or(W, 0x00F000F0u, kMagic), s16, o16);
            pr[4 * i + 2] = h2_sub(lop_and_or(W8, 0x000F000Fu, kMagic), sub);
            pr[4 * i + 3] = h2_fma(lop_and_or(W8, 0x00F000F0u, kMagic), s16, o16);
        }
    }
};

// 2-bit fields j = 0..3 of a byte pair: value 1024 + e * 4^j, q = e - off.
template <int OFF>
__device__ __forceinline__ uint32_t dec2(uint32_t x, int j) {
    const float m = float(1 << (2 * j));
    return h2_fma(lop_and_or(x, 0x00030003u << (2 * j), kMagic), h2c(1.0f / m), h2c(-(1024.0f / m + OFF)));
}

template <>
struct KUnpack<2> {
    static constexpr int kSliceBytes = 8;
    __device__ static int ca(int p) { return 16 * (p >> 3) + (p & 7); }
    __device__ static int cb(int p) { return ca(p) + 8; }
    __device__ static void run(const uint8_t* row, int t, uint32_t (&pr)[16]) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * t);
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                pr[8 * i + j] = dec2<2>(w[i], j);
                pr[8 * i + 4 + j] = dec2<2>(w[i] >> 8, j);
            }
        }
    }
};

template <>
struct KUnpack<3> {
    static constexpr int kSliceBytes = 8;  // low 2-bit plane; plus 4 bytes of the high plane
    __device__ static int ca(int p) { return 16 * (p >> 3) + (p & 7); }
    __device__ static int cb(int p) { return ca(p) + 8; }
    __device__ static void run(const uint8_t* row, int t, uint32_t (&pr)[16]) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * t);
        const uint32_t H = *reinterpret_cast<const uint32_t*>(row + 32 + 4 * t);
        const uint32_t w[2] = {v.x, v.y};
        const uint32_t one = 0x3C003C00u, four = h2c(4.0f);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t lo = dec2<4>(j < 4 ? w[i] : (w[i] >> 8), j & 3);  // e_lo - 4
                // high bits of channels 16i + j and 16i + j + 8 -> fp16x2 0/1
                const uint32_t hb = prmt((H >> (16 * i + j)) & 0x101u, 0u, 0x4140u);
                const uint32_t hf = h2_sub(hb | kMagic, h2c(1024.0f));
                (void)one;
                pr[8 * i + j] = h2_fma(hf, four, lo);
            }
        }
    }
};

// V side.  Thread g of a warp owns channels [16g, 16g + 16) of a token row.
// For two token rows r0, r1 it produces the 16 fp16x2 values
// (code[r0][c], code[r1][c]) for c = 16g + k, k = 0..15, in pr[k].
template <int BITS>
struct VUnpack;

template <>
struct VUnpack<4> {
    __device__ static void run(const uint8_t* r0, const uint8_t* r1, int g, uint32_t (&pr)[16]) {
        const uint2 u0 = *reinterpret_cast<const uint2*>(r0 + 8 * g);
        const uint2 u1 = *reinterpret_cast<const uint2*>(r1 + 8 * g);
        const uint32_t sub = h2c(1032.0f), s16 = h2c(1.0f / 16.0f), o16 = h2c(-72.0f);
        const uint32_t a[2] = {u0.x, u0.y}, b[2] = {u1.x, u1.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                // bytes 2hh, 2hh+1 of both rows: channels 8i + 4hh .. + 3
                const uint32_t x = prmt(a[i], b[i], hh ? 0x7632u : 0x5410u);
                const uint32_t x8 = x >> 8;
                const int k = 8 * i + 4 * hh;
                pr[k + 0] = h2_sub(lop_and_or(x, 0x000F000Fu, kMagic), sub);
                pr[k + 1] = h2_fma(lop_and_or(x, 0x00F000F0u, kMagic), s16, o16);
                pr[k + 2] = h2_sub(lop_and_or(x8, 0x000F000Fu, kMagic), sub);
                pr[k + 3] = h2_fma(lop_and_or(x8, 0x00F000F0u, kMagic), s16, o16);
            }
        }
    }
};

template <>
struct VUnpack<2> {
    __device__ static void run(const uint8_t* r0, const uint8_t* r1, int g, uint32_t (&pr)[16]) {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(r0 + 4 * g);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(r1 + 4 * g);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t x = prmt(a, b, hh ? 0x7632u : 0x5410u);  // channels 8hh .. 8hh + 7
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                pr[8 * hh + j] = dec2<2>(x, j);
                pr[8 * hh + 4 + j] = dec2<2>(x >> 8, j);
            }
        }
    }
};

template <>
struct VUnpack<3> {
    __device__ static void run(const uint8_t* r0, const uint8_t* r1, int g, uint32_t (&pr)[16]) {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(r0 + 4 * g);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(r1 + 4 * g);
        const uint32_t ha = *reinterpret_cast<const uint16_t*>(r0 + 32 + 2 * g);
        const uint32_t hb = *reinterpret_cast<const uint16_t*>(r1 + 32 + 2 * g);
        const uint32_t hh2 = ha | (hb << 16);  // bit k: row 0 channel k; bit 16 + k: row 1 channel k
        const uint32_t four = h2c(4.0f);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t x = prmt(a, b, hh ? 0x7632u : 0x5410u);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = 8 * hh + j;
                const uint32_t lo = dec2<4>(j < 4 ? x : (x >> 8), j & 3);
                const uint32_t hf = h2_sub(((hh2 >> k) & 0x00010001u) | kMagic, h2c(1024.0f));
                pr[k] = h2_fma(hf, four, lo);
            }
        }
    }
};

// ---------------------------------------------------------------- slot layout

template <int D, int BITS, int MODE>
struct SlotLayout {
    static constexpr int kRB = D * BITS / 8;
    static constexpr int kNtok = (MODE == kNsn) ? 2 : 1;
    static constexpr int kCodes = 0;
    static constexpr int kTok = kT * kRB;
    static constexpr int kChan = kTok + kT * kNtok * 2;
    static constexpr int kOff = kChan + ((MODE != kNaive) ? D * 2 : 0);
    static constexpr int kBytes = kOff + ((MODE == kNsn) ? D * 2 : 0);
    static constexpr int kStride = (kBytes + 127) / 128 * 128;
};

// Merge buffers reuse the ring after every warp is done with it.
template <int D>
__host__ __device__ constexpr int mma_merge_bytes() {
    return (2 * kNW * kGMax + 2 * kNW * kGMax * D + kGMax * kT + 2 * kGMax) * 4;
}

template <int D, int BITS, int MODE>
__host__ __device__ constexpr int mma_smem_bytes() {
    constexpr int ring = kNW * kRing * SlotLayout<D, BITS, MODE>::kStride + kNW * kRing * 8;
    constexpr int merge = mma_merge_bytes<D>();
    return (ring > merge ? ring : merge) + 128;
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- the kernel

// GP: padded heads per kv head, 4 (G <= 4: one n-tile holds hi and lo of four
// heads) or 8 (G <= 8: hi and lo n-tiles of eight heads).
template <int D, int BITS, int MODE, bool HAD, int GP>
__global__ void __launch_bounds__(kNW * 32) decode_mma_kernel(DecodeArgs a) {
    static_assert(D == 128, "tensor-core decode is built for head dim 128");
    using SL = SlotLayout<D, BITS, MODE>;
    constexpr int NTS = 2 * GP / 8;       // score n-tiles (1 or 2)
    constexpr int NCOL = (GP == 4) ? 2 : 2;  // heads held per thread
    constexpr bool PCH = MODE != kNaive;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int QMAX = (1 << (BITS - 1)) - 1;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int G = a.G;
    const int b = bh / a.H, h = bh % a.H;
    const int nb_cap = a.cap / kT;

    uint8_t* ring = smem_raw;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kNW * kRing * SL::kStride);
    __shared__ float s_q[kGMax][D];  // queries (original domain)
    __shared__ float s_qt[kGMax][D]; // queries, rotated domain (== s_q without HADAMARD)
    __shared__ float s_qscale[kGMax];

    // ---- prologue: queries, rotation, per-head power-of-two scale
    for (int i = tid; i < kGMax * D; i += kNW * 32) {
        const int j = i / D, c = i % D;
        float qv = 0.0f;
        if (j < G) qv = __half2float(a.q[((size_t)b * a.H * G + (size_t)h * G + j) * D + c]);
        s_q[j][c] = qv;
        s_qt[j][c] = qv;
    }
    if (tid < kNW * kRing) mbar_init(&bars[tid], 1);
    fence_mbar_init();
    __syncthreads();
    if (tid < kGMax) {
        float r[D];
#pragma unroll
        for (int c = 0; c < D; ++c) r[c] = s_q[tid][c];
        if constexpr (HAD) {
#pragma unroll
            for (int c = 0; c < D; ++c)
                if (a.signs != nullptr && a.signs[c] < 0) r[c] = -r[c];
            fwht_reg<D>(r);
#pragma unroll
            for (int c = 0; c < D; ++c) s_qt[tid][c] = r[c];
        }
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < D; ++c) amax = fmaxf(amax, fabsf(r[c]));
        // |q'| <= amax * max(sigma) <= amax / qmax (1 + 2^-10); keep it <= 2^13
        const float bound = PCH ? amax * (1.001f / (float)QMAX) : amax;
        s_qscale[tid] = bound > 0.0f ? pow2i(13 - ceil_log2(bound)) : 1.0f;
    }
    __syncthreads();

    // ---- this warp's blocks
    const int blk_begin = split * a.bps;
    const int blk_end = min(a.nbq, blk_begin + a.bps);
    const int nmine = blk_end > blk_begin + warp ? (blk_end - blk_begin - warp + kNW - 1) / kNW : 0;
    const int nunits = 2 * nmine;
    uint8_t* my_ring = ring + warp * kRing * SL::kStride;
    uint64_t* my_bars = bars + warp * kRing;

    auto issue = [&](int u) {
        // unit u: block blk_begin + warp + kNW * (u / 2), tensor u % 2
        const int blk = blk_begin + warp + kNW * (u >> 1);
        const int ten = u & 1;
        uint8_t* slot = my_ring + (u % kRing) * SL::kStride;
        uint64_t* bar = &my_bars[u % kRing];
        const size_t row0 = (size_t)bh * a.cap + (size_t)blk * kT;
        const size_t bi = ((size_t)bh * nb_cap + blk) * D;
        mbar_expect_tx(bar, SL::kBytes);
        bulk_load(slot + SL::kCodes, (ten ? a.codes[1] : a.codes[0]) + row0 * SL::kRB, kT * SL::kRB, bar);
        bulk_load(slot + SL::kTok, (ten ? a.tok[1] : a.tok[0]) + row0 * SL::kNtok, kT * SL::kNtok * 2, bar);
        if (PCH) bulk_load(slot + SL::kChan, (ten ? a.chan[1] : a.chan[0]) + bi, D * 2, bar);
        if (MODE == kNsn) bulk_load(slot + SL::kOff, (ten ? a.off[1] : a.off[0]) + bi, D * 2, bar);
    };
    int issued = min(kRing, nunits);  // units issued so far (same value in every lane)
    if (lane == 0) {
        for (int u = 0; u < issued; ++u) issue(u);
    }
    int waited = 0;  // units whose slot phase this warp has seen complete

    // per-thread persistent state
    // heads held by this thread in the score / value layouts
    const int hbase = (GP == 4) ? 2 * (t & 1) : 2 * t;
    float m_run[NCOL], l_run[NCOL];
#pragma unroll
    for (int k = 0; k < NCOL; ++k) { m_run[k] = -INFINITY; l_run[k] = 0.0f; }
    float acc[NTS][8][4];
#pragma unroll
    for (int n = 0; n < NTS; ++n)
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[n][i][k] = 0.0f;
    // NSN mean term: lane owns channels 4*lane .. 4*lane+3 for all heads
    float acco[GP][4];
#pragma unroll
    for (int j = 0; j < GP; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) acco[j][k] = 0.0f;
    // rotated queries of the score column(s) this thread feeds, at its 32 channels
    // (GP == 4: column g -> head g & 3, part g >> 2; GP == 8: head g, both parts)
    const int qhead = (GP == 4) ? (g & 3) : g;
    const bool qlo = (GP == 4) && (g >= 4);
    const float* qt_row = &s_qt[qhead][32 * t];
    const float qsc = s_qscale[qhead];
    float qsc_col[NCOL];
#pragma unroll
    for (int k = 0; k < NCOL; ++k) qsc_col[k] = 1.0f / s_qscale[hbase + k];

    const float alpha2 = a.scale * kLog2e;
    bool ok = true;

    for (int it = 0; it < nmine; ++it) {
        const int uK = 2 * it, uV = 2 * it + 1;
        uint8_t* sk = my_ring + (uK % kRing) * SL::kStride;
        uint8_t* sv = my_ring + (uV % kRing) * SL::kStride;
        // ---------------- K half
        if (!mbar_wait(&my_bars[uK % kRing], (uK / kRing) & 1, 1u << 26)) { ok = false; break; }
        waited = uK + 1;
        // B fragments: q' = qt * sigma^K * 2^e, as fp16 hi (and lo) parts
        uint32_t bq[NTS][16];
        {
            const __half* sig = reinterpret_cast<const __half*>(sk + SL::kChan) + 32 * t;
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int ca = KUnpack<BITS>::ca(p), cb = KUnpack<BITS>::cb(p);
                const float fa = qt_row[ca] * (PCH ? __half2float(sig[ca]) : 1.0f) * qsc;
                const float fb = qt_row[cb] * (PCH ? __half2float(sig[cb]) : 1.0f) * qsc;
                const __half ha = __float2half_rn(fa), hb = __float2half_rn(fb);
                const float ra = fa - __half2float(ha), rb = fb - __half2float(hb);
                if constexpr (GP == 4) {
                    bq[0][p] = qlo ? pack_h2(ra, rb) : pack_h2(__half2float(ha), __half2float(hb));
                } else {
                    bq[0][p] = pack_h2(__half2float(ha), __half2float(hb));
                    bq[1][p] = pack_h2(ra, rb);
                }
            }
        }
        // scores for 8 m-tiles of 16 tokens
        float sc[8][4];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pa[16], pb[16];
            KUnpack<BITS>::run(sk + SL::kCodes + (16 * mt + g) * SL::kRB, t, pa);
            KUnpack<BITS>::run(sk + SL::kCodes + (16 * mt + g + 8) * SL::kRB, t, pb);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma16816(d0, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], bq[0][2 * s], bq[0][2 * s + 1]);
                if constexpr (NTS == 2)
                    mma16816(d1, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], bq[1][2 * s], bq[1][2 * s + 1]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if constexpr (GP == 4) sc[mt][k] = d0[k] + __shfl_xor_sync(0xffffffffu, d0[k], 2);
                else sc[mt][k] = d0[k] + d1[k];
            }
        }
        // per-token K factors, logits (log2 domain)
        const __half* tk = reinterpret_cast<const __half*>(sk + SL::kTok);
        float qoK[NCOL];
        if constexpr (MODE == kNsn) {
            // q . o^K for this thread's heads (lanes own 4 channels each)
            const __half* ok_ = reinterpret_cast<const __half*>(sk + SL::kOff);
            float part[GP];
#pragma unroll
            for (int j = 0; j < GP; ++j) {
                float s = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) s += s_q[j][4 * lane + k] * __half2float(ok_[4 * lane + k]);
                part[j] = s;
            }
#pragma unroll
            for (int j = 0; j < GP; ++j)
#pragma unroll
                for (int o = 16; o; o >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
#pragma unroll
            for (int k = 0; k < NCOL; ++k) {
                float v = 0.0f;
#pragma unroll
                for (int j = 0; j < GP; ++j)
                    if (j == hbase + k) v = part[j];
                qoK[k] = v;
            }
        }
        float bmax[NCOL] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int tok = 16 * mt + g + 8 * r;
                float kap, add = 0.0f;
                if constexpr (MODE == kNsn) {
                    const __half2 s12 = reinterpret_cast<const __half2*>(tk)[tok];
                    const float s1 = __low2float(s12), s2 = __high2float(s12);
                    kap = s1 * s2 * (HAD ? 1.0f : a.sqd);
                    add = s1;
                } else {
                    kap = __half2float(tk[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                }
#pragma unroll
                for (int k = 0; k < NCOL; ++k) {
                    float lg = sc[mt][2 * r + k] * (kap * qsc_col[k]);
                    if constexpr (MODE == kNsn) lg += add * qoK[k];
                    lg *= alpha2;
                    sc[mt][2 * r + k] = lg;
                    bmax[k] = fmaxf(bmax[k], lg);
                }
            }
        }
        // K slot consumed: reuse it for the unit kRing ahead
        __syncwarp();
        if (uK + kRing < nunits) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(uK + kRing);
            }
            issued = uK + kRing + 1;
        }
#pragma unroll
        for (int k = 0; k < NCOL; ++k) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) bmax[k] = fmaxf(bmax[k], __shfl_xor_sync(0xffffffffu, bmax[k], o));
        }
        // ---------------- V half
        if (!mbar_wait(&my_bars[uV % kRing], (uV / kRing) & 1, 1u << 26)) { ok = false; break; }
        waited = uV + 1;
        const __half* tv = reinterpret_cast<const __half*>(sv + SL::kTok);
        // online softmax update
        float corr[NCOL];
        bool changed = false;
#pragma unroll
        for (int k = 0; k < NCOL; ++k) {
            const float mn = fmaxf(m_run[k], bmax[k]);
            corr[k] = fast_exp2(m_run[k] - mn);  // 0 on the first block
            changed |= (mn != m_run[k]);
            m_run[k] = mn;
            l_run[k] *= corr[k];
        }
        if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
            for (int n = 0; n < NTS; ++n)
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[n][i][k] *= corr[k & 1];
            if constexpr (MODE == kNsn) {
                // correction of head j lives in lane t = (j / 2) mod 2 (GP 4) or j / 2 (GP 8)
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                    const int src = (GP == 4) ? ((j >> 1) & 1) : (j >> 1);
                    const float cj = __shfl_sync(0xffffffffu, corr[j & 1], src);
#pragma unroll
                    for (int k = 0; k < 4; ++k) acco[j][k] *= cj;
                }
            }
        }
        // nu per token and the block's power-of-two scale for P'
        auto nu_of = [&](int tok, float& s1o) -> float {
            if constexpr (MODE == kNsn) {
                const __half2 s12 = reinterpret_cast<const __half2*>(tv)[tok];
                s1o = __low2float(s12);
                return __low2float(s12) * __high2float(s12) * (HAD ? 1.0f : a.sqd);
            } else {
                s1o = 0.0f;
                return __half2float(tv[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
            }
        };
        float numax = 0.0f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float s1o;
                numax = fmaxf(numax, nu_of(16 * mt + g + 8 * r, s1o));
            }
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) numax = fmaxf(numax, __shfl_xor_sync(0xffffffffu, numax, o));
        const int fexp = numax > 0.0f ? 13 - ceil_log2(numax) : 0;
        const float pscale = pow2i(fexp), pinv = pow2i(-fexp);
        // values: P' fragments via movmatrix, V codes transposed
        float dv[NTS][8][4];
#pragma unroll
        for (int n = 0; n < NTS; ++n)
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) dv[n][i][k] = 0.0f;
        float lsum[NCOL] = {0.f, 0.f}, bsum[NCOL] = {0.f, 0.f};
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t prow[NTS][2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float pv[NCOL], s1o;
                const float nus = nu_of(16 * mt + g + 8 * r, s1o) * pscale;
#pragma unroll
                for (int k = 0; k < NCOL; ++k) {
                    const float p = fast_exp2(sc[mt][2 * r + k] - m_run[k]);
                    lsum[k] += p;
                    if constexpr (MODE == kNsn) bsum[k] += p * s1o;
                    pv[k] = p * nus;
                }
                const __half h0 = __float2half_rn(pv[0]), h1 = __float2half_rn(pv[1]);
                const float l0 = pv[0] - __half2float(h0), l1 = pv[1] - __half2float(h1);
                if constexpr (GP == 4) {
                    prow[0][r] = (t >= 2) ? pack_h2(l0, l1) : pack_h2(__half2float(h0), __half2float(h1));
                } else {
                    prow[0][r] = pack_h2(__half2float(h0), __half2float(h1));
                    prow[1][r] = pack_h2(l0, l1);
                }
            }
            uint32_t bp[NTS][2];
#pragma unroll
            for (int n = 0; n < NTS; ++n) {
                bp[n][0] = movmatrix_t(prow[n][0]);
                bp[n][1] = movmatrix_t(prow[n][1]);
            }
            // V rows of this 16-token tile: (2t, 2t+1) and (2t+8, 2t+9)
            uint32_t va[16], vb[16];
            const uint8_t* vbase = sv + SL::kCodes + (16 * mt) * SL::kRB;
            VUnpack<BITS>::run(vbase + (2 * t) * SL::kRB, vbase + (2 * t + 1) * SL::kRB, g, va);
            VUnpack<BITS>::run(vbase + (2 * t + 8) * SL::kRB, vbase + (2 * t + 9) * SL::kRB, g, vb);
#pragma unroll
            for (int tc = 0; tc < 8; ++tc) {
#pragma unroll
                for (int n = 0; n < NTS; ++n)
                    mma16816(dv[n][tc], va[2 * tc], va[2 * tc + 1], vb[2 * tc], vb[2 * tc + 1], bp[n][0], bp[n][1]);
            }
        }
#pragma unroll
        for (int k = 0; k < NCOL; ++k) l_run[k] += lsum[k];
        // block scale: acc[c][col] += dv * sigma^V_c * 2^-fexp
        {
            const __half* sigv = reinterpret_cast<const __half*>(sv + SL::kChan) + 16 * g;
#pragma unroll
            for (int tc = 0; tc < 8; ++tc) {
                const float s0 = (PCH ? __half2float(sigv[2 * tc]) : 1.0f) * pinv;
                const float s1_ = (PCH ? __half2float(sigv[2 * tc + 1]) : 1.0f) * pinv;
#pragma unroll
                for (int n = 0; n < NTS; ++n) {
                    acc[n][tc][0] += dv[n][tc][0] * s0;
                    acc[n][tc][1] += dv[n][tc][1] * s0;
                    acc[n][tc][2] += dv[n][tc][2] * s1_;
                    acc[n][tc][3] += dv[n][tc][3] * s1_;
                }
            }
        }
        if constexpr (MODE == kNsn) {
            // beta_j = sum over the block of p * s1 (scores of head j live in lanes with t = hbase/2)
#pragma unroll
            for (int k = 0; k < NCOL; ++k)
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) bsum[k] += __shfl_xor_sync(0xffffffffu, bsum[k], o);
            const __half* ov = reinterpret_cast<const __half*>(sv + SL::kOff);
#pragma unroll
            for (int j = 0; j < GP; ++j) {
                const int src = (GP == 4) ? ((j >> 1) & 1) : (j >> 1);
                const float bj = __shfl_sync(0xffffffffu, bsum[j & 1], src);
#pragma unroll
                for (int k = 0; k < 4; ++k) acco[j][k] += bj * __half2float(ov[4 * lane + k]);
            }
        }
        __syncwarp();
        if (uV + kRing < nunits) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(uV + kRing);
            }
            issued = uV + kRing + 1;
        }
    }
    if (!ok) {
        // give the copies still in flight a bounded time to land before the
        // shared memory is reused; the results of this call are void
        if (lane == 0) report_error(kErrBarrierTimeout);
        for (int u = waited; u < issued; ++u) mbar_wait(&my_bars[u % kRing], (u / kRing) & 1, 1u << 20);
    }
    __syncwarp();
    if (lane == 0) {
        for (int i = 0; i < kRing; ++i) mbar_inval(&my_bars[i]);
    }

    // ---- merge: warps -> shared memory -> one partial per CTA
    // reduce l over the 8 row groups; combine hi + lo value columns
#pragma unroll
    for (int k = 0; k < NCOL; ++k)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) l_run[k] += __shfl_xor_sync(0xffffffffu, l_run[k], o);
    float accv[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if constexpr (GP == 4) accv[i][k] = acc[0][i][k] + __shfl_xor_sync(0xffffffffu, acc[0][i][k], 2);
            else accv[i][k] = acc[0][i][k] + acc[1][i][k];
        }
    __syncthreads();  // every warp is done with its ring; reuse it for the merge
    float* mw = reinterpret_cast<float*>(smem_raw);   // [kNW][kGMax] running max
    float* lw = mw + kNW * kGMax;                     // [kNW][kGMax] sums
    float* aw = lw + kNW * kGMax;                     // [kNW][kGMax][D] code-term accumulators
    float* ow = aw + kNW * kGMax * D;                 // [kNW][kGMax][D] original-domain accumulators
    if (g == 0 && (GP == 8 || t < 2)) {
#pragma unroll
        for (int k = 0; k < NCOL; ++k) {
            mw[warp * kGMax + hbase + k] = m_run[k];
            lw[warp * kGMax + hbase + k] = l_run[k];
        }
    }
    if (GP == 8 || t < 2) {
#pragma unroll
        for (int tc = 0; tc < 8; ++tc)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c = 16 * g + 2 * tc + (k >> 1);
                const int head = hbase + (k & 1);
                aw[(warp * kGMax + head) * D + c] = accv[tc][k];
            }
    }
#pragma unroll
    for (int j = 0; j < kGMax; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) ow[(warp * kGMax + j) * D + 4 * lane + k] = (j < GP) ? acco[j < GP ? j : 0][k] : 0.0f;
    __syncthreads();

    // residual tokens (fp16), handled by the last split on CUDA cores
    float* pp = a.part + ((size_t)bh * a.nsplit + split) * G * (2 + 2 * D);
    const bool do_res = (split == a.nsplit - 1) && a.rlen > 0;
    float* rl = ow + kNW * kGMax * D;  // [kGMax][kT] residual logits / weights
    float* rm = rl + kGMax * kT;       // [kGMax] residual max, [kGMax] sum
    if (do_res) {
        const __half* rk = a.resid[0] + (size_t)bh * kT * D;
        for (int i = tid; i < kGMax * kT; i += kNW * 32) {
            const int j = i / kT, tr = i % kT;
            float s = -INFINITY;
            if (j < G && tr < a.rlen) {
                s = 0.0f;
                for (int c = 0; c < D; ++c) s += s_q[j][c] * __half2float(rk[(size_t)tr * D + c]);
                s *= alpha2;
            }
            rl[i] = s;
        }
        __syncthreads();
        for (int j = warp; j < kGMax; j += kNW) {
            float mx = -INFINITY;
            for (int i = lane; i < kT; i += 32) mx = fmaxf(mx, rl[j * kT + i]);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float sm = 0.0f;
            for (int i = lane; i < kT; i += 32) {
                const float p = (mx == -INFINITY || rl[j * kT + i] == -INFINITY) ? 0.0f : fast_exp2(rl[j * kT + i] - mx);
                rl[j * kT + i] = p;
                sm += p;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
            if (lane == 0) { rm[j] = mx; rm[kGMax + j] = sm; }
        }
        __syncthreads();
    }
    // final merge of the kNW warp states (+ residual) for head j, channel c
    const __half* rv = a.resid[1] + (size_t)bh * kT * D;
    for (int i = tid; i < G * D; i += kNW * 32) {
        const int j = i / D, c = i % D;
        float M = -INFINITY;
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, mw[w * kGMax + j]);
        if (do_res) M = fmaxf(M, rm[j]);
        float L = 0.0f, A = 0.0f, AO = 0.0f;
        for (int w = 0; w < kNW; ++w) {
            const float mwj = mw[w * kGMax + j];
            const float wt = (mwj == -INFINITY) ? 0.0f : fast_exp2(mwj - M);
            L += wt * lw[w * kGMax + j];
            A += wt * aw[(w * kGMax + j) * D + c];
            AO += wt * ow[(w * kGMax + j) * D + c];
        }
        if (do_res && rm[j] != -INFINITY) {
            const float wt = fast_exp2(rm[j] - M);
            L += wt * rm[kGMax + j];
            float s = 0.0f;
            for (int tr = 0; tr < a.rlen; ++tr) s += rl[j * kT + tr] * __half2float(rv[(size_t)tr * D + c]);
            AO += wt * s;
        }
        float* pj = pp + (size_t)j * (2 + 2 * D);
        // partial in natural-log units for the combine kernel
        if (c == 0) { pj[0] = (M == -INFINITY) ? -INFINITY : M * (1.0f / kLog2e); pj[1] = L; }
        pj[2 + c] = A;
        pj[2 + D + c] = AO;
    }
}

}  // namespace kvq
