// kvq_quant_rows.cuh -- the per-token quantizer that one CTA of 128 threads
// runs over a 128-token block (one thread per token row, the row in
// registers as packed fp32 pairs), and the packing of its codes.
//
// Arithmetic that decides a stored bit (norms, means, scales, codes) uses
// explicitly rounded operations (the _rn intrinsics, PTX .rn forms) so that
// the compiler never contracts or reorders it.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// ---------------------------------------------------------------- packed fp32 pairs
// sm_100 executes add/sub/mul/fma on two fp32 lanes per instruction
// (.f32x2); every lane is rounded exactly like the scalar instruction, so
// the packed forms change only the instruction count, never a result.  The
// quantizer keeps a token row as D/2 pairs P[j] = (channel j, channel
// j + D/2).
using f2_t = unsigned long long;

__device__ __forceinline__ f2_t f2_pack(float lo, float hi) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(f2_t x, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
    f2_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2_t f2_sub(f2_t a, f2_t b) {
    f2_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
    f2_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
    f2_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Lane-wise product rounded to fp32 on its own.  The assembler may fuse a
// packed mul.rn.f32x2 with the add or subtract that consumes it into one
// fused multiply-add (one rounding instead of two), and it also did so for
// an FMA whose addend was the literal -0.  So the product is an FMA whose
// addend nz is the pair (-0, -0) loaded from constant memory, a value the
// assembler cannot assume: a * b + (-0) rounds the exact product once (zero
// signs included), and an FMA is not fused again.  Every product that feeds
// an add whose operands are not exact products uses this.
__constant__ float g_neg_zero[2] = {-0.0f, -0.0f};

__device__ __forceinline__ f2_t neg_zero2() { return *reinterpret_cast<const f2_t*>(g_neg_zero); }

__device__ __forceinline__ f2_t f2_mul_sep(f2_t a, f2_t b, f2_t nz) {
    f2_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(nz));
    return r;
}

// Pairwise sum of squares over the pairs P[OFF .. OFF+N): lane 0 sums the
// first half of the row, lane 1 the second, with the same recursive halving.
// The volatile forms keep the depth-first order of the tree, so that the
// squares are not all formed (and held) before the first sums.
__device__ __forceinline__ f2_t f2_mul_ordered(f2_t a, f2_t b) {
    f2_t r;
    asm volatile("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2_t f2_add_ordered(f2_t a, f2_t b) {
    f2_t r;
    asm volatile("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// EXACT: the squares are exact in fp32 (values widened from fp16), so a
// fused square-and-add rounds like the separate operations and the packed
// multiply may be used; otherwise the squares are rounded on their own.
template <int OFF, int N, int H2, bool EXACT>
__device__ __forceinline__ f2_t pw_sumsq2(const f2_t (&P)[H2], f2_t nz) {
    if constexpr (N == 1) return EXACT ? f2_mul_ordered(P[OFF], P[OFF]) : f2_mul_sep(P[OFF], P[OFF], nz);
    else
        return f2_add_ordered(pw_sumsq2<OFF, N / 2, H2, EXACT>(P, nz), pw_sumsq2<OFF + N / 2, N / 2, H2, EXACT>(P, nz));
}

// Pairwise sum of squares of the whole row: the top split of the halving
// tree adds the two lanes.  nz: see f2_mul_sep (unused when EXACT).
template <int H2, bool EXACT>
__device__ __forceinline__ float row_sumsq(const f2_t (&P)[H2], f2_t nz) {
    float lo, hi;
    f2_unpack(pw_sumsq2<0, H2, H2, EXACT>(P, nz), lo, hi);
    return __fadd_rn(lo, hi);
}

// x_lo^2 + x_hi^2 of the two fp16 values of a word, rounded once to fp32:
// the square of an fp16 value is exact in fp32, so two mixed-precision fused
// multiply-adds (fp16 factors, fp32 addend) give exactly the fp32 sum of the
// two exact squares.
__device__ __forceinline__ float sumsq_h2(uint32_t w) {
    float r;
    asm volatile(
        "{\n .reg .b16 l, h;\n .reg .f32 s;\n mov.b32 {l, h}, %1;\n"
        " fma.rn.f32.f16 s, l, l, 0f00000000;\n fma.rn.f32.f16 %0, h, h, s;\n}"
        : "=f"(r)
        : "r"(w));
    return r;
}

// The pairwise sum of squares of pw_sumsq2 taken straight from the raw fp16
// row (chunk q = channels 8q .. 8q + 7): node OFF of the level above the
// squares sums channels 2 OFF, 2 OFF + 1 of the low half (lane 0) and of the
// high half (lane 1).
template <int OFF, int N, int D>
__device__ __forceinline__ f2_t raw_pw_sumsq(const uint4 (&raw)[D / 8]) {
    if constexpr (N == 1) {
        const uint32_t* lo = reinterpret_cast<const uint32_t*>(&raw[OFF / 4]);
        const uint32_t* hi = reinterpret_cast<const uint32_t*>(&raw[D / 16 + OFF / 4]);
        return f2_pack(sumsq_h2(lo[OFF % 4]), sumsq_h2(hi[OFF % 4]));
    } else {
        return f2_add_ordered(raw_pw_sumsq<OFF, N / 2, D>(raw), raw_pw_sumsq<OFF + N / 2, N / 2, D>(raw));
    }
}

template <int D>
__device__ __forceinline__ float raw_row_sumsq(const uint4 (&raw)[D / 8]) {
    float lo, hi;
    f2_unpack(raw_pw_sumsq<0, D / 4, D>(raw), lo, hi);
    return __fadd_rn(lo, hi);
}

// Butterflies of stride S (channels j, j + S inside each half), ascending.
template <int S, int H2>
__device__ __forceinline__ void fwht2_stage(f2_t (&P)[H2]) {
#pragma unroll
    for (int i = 0; i < H2; i += 2 * S) {
#pragma unroll
        for (int j = 0; j < S; ++j) {
            const f2_t a = P[i + j], b = P[i + j + S];
            P[i + j] = f2_add(a, b);
            P[i + j + S] = f2_sub(a, b);
        }
    }
    if constexpr (2 * S < H2) fwht2_stage<2 * S, H2>(P);
}

// Unnormalized Walsh-Hadamard transform of the row, strides 1, 2, ..., D/2
// in that order; the last stride pairs the two lanes of each P[j].
template <int H2>
__device__ __forceinline__ void fwht2(f2_t (&P)[H2]) {
    fwht2_stage<1, H2>(P);
#pragma unroll
    for (int j = 0; j < H2; ++j) {
        float a, b;
        f2_unpack(P[j], a, b);
        P[j] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
}

__device__ __forceinline__ uint32_t prmt32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// ---------------------------------------------------------------- the quantizer

// NSN block means: from the fp16 tile with the row still in its fp16 form
// (two tile regions, three CTAs per SM), or from the fp32 rows through a
// transposed buffer (three regions, two CTAs per SM).
#ifndef KVQ_NSN_TILE_MEANS
#define KVQ_NSN_TILE_MEANS 1
#endif
constexpr bool kNsnTileMeans = KVQ_NSN_TILE_MEANS != 0;

// Bytes of the per-token-group partials: the NSN column sums are
// (128 / (D / 8)) groups x D floats, the per-channel maxima half of that.
constexpr int kGpartBytes = 4096 + 512;  // group sums / warp maxima, then the DQ scratch

// Output pointers of one (tensor, batch, head, block).
struct QuantOut {
    uint8_t* codes;  // [128][row_bytes] rows of this block
    uint8_t* stage;  // if set, codes go here instead, for a TMA store: row t at t * row_bytes,
                     // 16-byte chunk c at chunk c ^ ((t >> 1) & 3) (INT4, 64-byte swizzle) or
                     // c ^ ((t >> 2) & 1) (INT2, 32-byte swizzle)
    __half* tok;     // [128][ntok]
    __half* chan;    // [D] (PER_CHANNEL)
    __half* off;     // [D] (NSN)
    bool pairv;      // V codes of head dim 128: pair-interleaved rows
};

// Shared-memory scratch of one quantizer CTA.
template <int D>
struct QuantSmem {
    // fp16 input tile: 64-channel boxes of 128 rows x 128 bytes, 16-byte
    // chunk c of row t stored at chunk c ^ (t & 7) (the TMA 128-byte swizzle)
    const uint8_t* tile;
    // NSN: fp32 [128][D] buffer of the rows in pair order, in two halves:
    // pairs [0, D/4) of every row in red_lo, pairs [D/4, D/2) in red_hi;
    // 16-byte chunk k of a half row t stored at chunk k ^ (t & (D/8 - 1))
    float* red_lo;
    float* red_hi;
    float* vec;      // [D] a per-channel vector in pair order (means, reciprocal scales)
    float* gpart;    // [4 KB] per-token-group partial sums (NSN means), then per-warp maxima
    float* tokv;     // [128] a per-token scalar (NSN 1/||x|| * sqrt(d))
    uint32_t* sgn2;  // [D/2] fp16x2 sign masks of channels (2i, 2i+1)
    QuantOut* out;   // the current block's output pointers
};

// Widen 8 fp16 channels of the low half (lo) and the matching 8 of the high
// half (hi) into pairs P[8q .. 8q+8), after the rotation's sign flips when
// SIGNS (the plain Hadamard transform has none).
template <int D, bool SIGNS>
__device__ __forceinline__ void widen_chunk(uint4 lo, uint4 hi, int q, const QuantSmem<D>& sm, f2_t (&P)[D / 2]) {
    if constexpr (SIGNS) {
        const uint4 ml = reinterpret_cast<const uint4*>(sm.sgn2)[q];
        const uint4 mh = reinterpret_cast<const uint4*>(sm.sgn2)[D / 16 + q];
        lo.x ^= ml.x; lo.y ^= ml.y; lo.z ^= ml.z; lo.w ^= ml.w;
        hi.x ^= mh.x; hi.y ^= mh.y; hi.z ^= mh.z; hi.w ^= mh.w;
    }
    const __half2* hl = reinterpret_cast<const __half2*>(&lo);
    const __half2* hh = reinterpret_cast<const __half2*>(&hi);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __half22float2(hl[i]), b = __half22float2(hh[i]);
        P[8 * q + 2 * i] = f2_pack(a.x, b.x);
        P[8 * q + 2 * i + 1] = f2_pack(a.y, b.y);
    }
}

// The row as pairs P[j] = (channel j, channel j + D/2) from its raw fp16
// chunks (chunk q = channels 8q .. 8q + 7).
template <int D, bool SIGNS>
__device__ __forceinline__ void widen_row(const uint4 (&raw)[D / 8], const QuantSmem<D>& sm, f2_t (&P)[D / 2]) {
#pragma unroll
    for (int q = 0; q < D / 16; ++q) widen_chunk<D, SIGNS>(raw[q], raw[D / 16 + q], q, sm, P);
}



// Words of token t's row_bytes half of its pair block (pair-interleaved V
// rows), exchanged with the partner token t ^ 1 (same warp; every lane
// calls this): token 2k + s takes units s W .. s W + W - 1 of both rows.
template <int BITS, int W>
__device__ __forceinline__ void pairv_words(int t, const uint32_t (&w)[W], uint32_t (&v)[W]) {
    static_assert(W % 2 == 0, "even number of words per row");
    const bool odd = (t & 1) != 0;
    // (row 2k unit, row 2k + 1 unit) from (own word, partner's word): the
    // even thread holds row 2k, the odd one row 2k + 1
    const uint32_t sel_lo = odd ? 0x1054u : 0x5410u, sel_hi = odd ? 0x3276u : 0x7632u;
#pragma unroll
    for (int j = 0; j < W / 2; ++j) {
        const uint32_t own = odd ? w[W / 2 + j] : w[j];  // units 2j, 2j + 1 of this half
        const uint32_t p = __shfl_xor_sync(0xffffffffu, odd ? w[j] : w[W / 2 + j], 1);
        v[2 * j] = prmt32(own, p, sel_lo);
        v[2 * j + 1] = prmt32(own, p, sel_hi);
    }
    if constexpr (BITS == 4) {
        static_assert(W == 16, "INT4 rows of head dim 128: four 16-byte chunks per half");
        // chunk c of the pair block at c ^ (2 (k & 1)): on odd pairs the
        // chunks 0, 1 of this half trade places with 2, 3
        if ((t >> 1) & 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t x = v[i];
                v[i] = v[i + 8];
                v[i + 8] = x;
            }
        }
    }
}

// Row t of packed codes: straight to global memory, or into the swizzled
// staging tile of a TMA store (then visible to the async proxy).
template <int D, int BITS>
__device__ __forceinline__ void store_codes(const QuantOut& out, int t, const uint32_t (&w0)[RowLayout<D, BITS>::kWords]) {
    using L = RowLayout<D, BITS>;
    uint32_t w[L::kWords];
#pragma unroll
    for (int i = 0; i < L::kWords; ++i) w[i] = w0[i];
    if constexpr (pairv_layout<D>()) {
        if (out.pairv) pairv_words<BITS, L::kWords>(t, w0, w);
    }
    if constexpr (BITS == 4 || BITS == 2) {
        if (out.stage != nullptr) {
            constexpr int NC = L::kBytes / 16;  // 16-byte chunks per row
            const int sw = (L::kBytes == 64) ? ((t >> 1) & 3) : ((t >> 2) & 1);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int pc = (c ^ sw) & (NC - 1);
                *reinterpret_cast<uint4*>(out.stage + (size_t)t * L::kBytes + pc * 16) =
                    make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
            fence_proxy_async_smem();
            return;
        }
    }
    store_words<L::kWords>(out.codes + (size_t)t * L::kBytes, w);
}

// Sign of channel c of the rotation as an fp16 sign-bit mask.
__device__ __forceinline__ uint16_t sign16(const uint32_t* sgn2, int c) {
    return (uint16_t)((sgn2[c >> 1] >> ((c & 1) * 16)) & 0x8000u);
}

// 16-byte shared-memory load of two pairs kept in program order (volatile),
// so that a loop of them does not have all its loads hoisted ahead of their
// uses.
__device__ __forceinline__ void lds_f2x2(uint32_t addr, f2_t& a, f2_t& b) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr));
}

// min / max over the warp's lanes of x (exact).
__device__ __forceinline__ float warp_min(float x) {
    float r;
    asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float warp_max(float x) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}

// max over the warp's lanes of |x| (exact: a comparison, no rounding).
__device__ __forceinline__ float warp_max_abs(float x) {
    float r;
    asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}

// Offset-binary code words of one pair: lanes of r = fma(x, inv, kC) with
// kC = 1.5 * 2^23 + 2^(BITS-1).  For any |rne(x * inv)| <= qmax the float
// lies in [2^23, 2^24), where its ulp is 1, so the single rounding of the
// fused product is round-half-even of x * inv (the added constant is even)
// and the low mantissa bits hold the offset-binary code e; the bits above
// the code (bit 22 upward) never reach the low 16 bits of the packing sums.
// Clamped to [-qmax, qmax] when CLAMP.
template <bool CLAMP>
__device__ __forceinline__ void code_pair(f2_t x, f2_t inv, float kQ, float kC, uint32_t& clo, uint32_t& chi) {
    float lo, hi;
    f2_unpack(f2_fma(x, inv, f2_pack(kC, kC)), lo, hi);
    if constexpr (CLAMP) {
        lo = fminf(fmaxf(lo, kC - kQ), kC + kQ);
        hi = fminf(fmaxf(hi, kC - kQ), kC + kQ);
    }
    clo = __float_as_uint(lo);
    chi = __float_as_uint(hi);
}

// Low 16 bits of sum_i e[i] << (NB * i) for N codes of NB bits (the bits of
// each word above bit 21 stay out of the low half, see code_pair).
template <int N, int NB>
__device__ __forceinline__ uint32_t pack_half(const uint32_t* e) {
    uint32_t h = e[0];
#pragma unroll
    for (int i = 1; i < N; ++i) h += e[i] << (NB * i);
    return h;
}

// Codes of the row held in registers (reciprocal scales in pair order in
// vec, or, when UNIFORM, one reciprocal scale inv for the whole row),
// packed as they are produced: a group of GP pairs gives GP codes of the
// low half (channels j ..) and GP of the high half (channels j + D/2 ..),
// folded at once into half-words (INT4 / INT2, and the 2-bit plane of INT3)
// or bytes (the bit plane of INT3), so that few code words are live while
// most of the row still is.
template <int D, int BITS, bool CLAMP, bool UNIFORM = false>
__device__ __forceinline__ void codes_from_regs(const f2_t (&P)[D / 2], const float* vec,
                                                uint32_t (&w)[RowLayout<D, BITS>::kWords], float inv = 0.0f) {
    using L = RowLayout<D, BITS>;
    constexpr int H2 = D / 2;
    constexpr float kQ = (float)L::kQmax;
    constexpr float kC = 12582912.0f + (float)L::kOff;
    constexpr int GP = (BITS == 4) ? 4 : 8;  // pairs per group: one half-word of codes per half
    const f2_t* iv = reinterpret_cast<const f2_t*>(vec);
    uint32_t pend_lo = 0, pend_hi = 0;  // the first half-words of the words being built
#pragma unroll
    for (int q = 0; q < H2 / GP; ++q) {
        uint32_t lo[GP], hi[GP];
#pragma unroll
        for (int i = 0; i < GP; i += 2) {
            ulonglong2 r;
            if constexpr (UNIFORM) r = make_ulonglong2(f2_pack(inv, inv), f2_pack(inv, inv));
            else r = *reinterpret_cast<const ulonglong2*>(iv + q * GP + i);
            code_pair<CLAMP>(P[q * GP + i], r.x, kQ, kC, lo[i], hi[i]);
            code_pair<CLAMP>(P[q * GP + i + 1], r.y, kQ, kC, lo[i + 1], hi[i + 1]);
        }
        uint32_t hl, hh;  // this group's half-words (16 bits of codes in the low half)
        if constexpr (BITS == 4) {
            hl = pack_half<4, 4>(lo);
            hh = pack_half<4, 4>(hi);
        } else if constexpr (BITS == 2) {
            hl = pack_half<8, 2>(lo);
            hh = pack_half<8, 2>(hi);
        } else {
            // the 2-bit plane (e & 3) and the bit plane (bit 2 of e)
            hl = 0; hh = 0;
            uint32_t bl = 0, bh = 0;
#pragma unroll
            for (int i = 0; i < GP; ++i) {
                hl |= (lo[i] & 3u) << (2 * i);
                hh |= (hi[i] & 3u) << (2 * i);
                bl |= ((lo[i] >> 2) & 1u) << i;
                bh |= ((hi[i] >> 2) & 1u) << i;
            }
            constexpr int BP = D / 16;  // first word of the bit plane
            const int sh = 8 * (q & 3);
            if ((q & 3) == 0) {
                w[BP + q / 4] = bl;
                w[BP + H2 / 32 + q / 4] = bh;
            } else {
                w[BP + q / 4] |= bl << sh;
                w[BP + H2 / 32 + q / 4] |= bh << sh;
            }
        }
        // two groups make a word: 8 INT4 codes, 16 INT2 codes or 16 2-bit fields
        constexpr int WH = (BITS == 4) ? H2 / 8 : H2 / 16;  // words of the low half
        if (q & 1) {
            w[q / 2] = prmt32(pend_lo, hl, 0x5410u);
            w[WH + q / 2] = prmt32(pend_hi, hh, 0x5410u);
        } else {
            pend_lo = hl;
            pend_hi = hh;
        }
    }
}

// Quantize the 128 token rows of one block.  Thread t (0..127) passes row t
// as its raw fp16 chunks (chunk q = channels 8q .. 8q + 7, without the
// rotation's signs) and works on it as pairs P[j] = (x[j], x[j + D/2]) in
// fp32, with the signs applied (SIGNS) when the pairs are formed; all 128
// threads of the CTA call this.
//   nsep:  n = ||x||, u = H(s (.) x) * (c0 / n)
//   NSN:   s1 = ||x|| rsqd, a = x (sqd / ||x||), o = block mean of a (fp16),
//          b = a - o, s2 = ||b|| rsqd, u = H(s (.) b) * (c0 / ||b||)
//   naive: u = x
// with c0 = rsqd under HADAMARD, else 1; then sigma = fp16(max|u| / qmax)
// per channel over the block (per token for naive) and codes
// rne(u * (1/sigma)) clamped.  Sign flips commute exactly with every step
// up to the rotation (means, norms, fp16 rounding are all sign-symmetric),
// which is why they can be applied when the row is loaded; the stored
// offsets are flipped back.  out gives the block's output pointers
// (built where they are used, to keep registers free).  The fp16 tile is
// last read before the barrier that publishes the NSN means; codes are
// staged (QuantOut::stage) only after a later barrier, so the staging tile
// may overlay the fp16 tile.
template <int D, int BITS, int MODE, bool HAD, bool SIGNS, typename Pre, typename Post>
__device__ __forceinline__ void quantize_rows(uint4 (&raw)[D / 8], const int t, const QuantSmem<D>& sm,
                                              const QuantOut& out, const float rsqd, const float sqd,
                                              Pre before_spill, Post after_means) {
    using L = RowLayout<D, BITS>;
    constexpr int H2 = D / 2;
    const float c0 = HAD ? rsqd : 1.0f;
    float kscale = 1.0f;
    f2_t P[H2];

    if constexpr (is_nsn(MODE)) {
        constexpr bool DQ = MODE == kNsnDq;
        const f2_t NZ = neg_zero2();
        // DQ scratch past the group sums (4 KB): [0, 4) warp minima of s1,
        // [4, 8) warp maxima, [8, 8 + D/32) warp maxima of |o|, then the o codes
        float* dqs = sm.gpart + 1024;
        uint8_t* dq_e = reinterpret_cast<uint8_t*>(dqs + 16);
        const float n1 = __fsqrt_rn(raw_row_sumsq<D>(raw));
        const float s1 = __fmul_rn(n1, rsqd);
        const float r1 = n1 > 0.0f ? __fdiv_rn(sqd, n1) : 0.0f;
        const f2_t R1 = f2_pack(r1, r1);
        if constexpr (DQ) {
            const float mn = warp_min(s1), mx = warp_max(s1);
            if ((t & 31) == 0) {
                dqs[t >> 5] = mn;
                dqs[4 + (t >> 5)] = mx;
            }
        }
        if constexpr (kNsnTileMeans) {
            // block means of a = x * r1 from the fp16 tile (unsigned values,
            // the same separately rounded products as the rows'), while the
            // row waits in its fp16 form: thread t sums the 8 channels of
            // chunk column kc8 over the TGC tokens of group gc in the
            // pairwise (binary-counter) order
            sm.tokv[t] = r1;
            __syncthreads();
            constexpr int NKC = D / 8, NGC = kT / NKC, TGC = kT / NGC;
            static_assert(NGC * D * 4 <= 4096, "group sums fit below the DQ scratch");
            constexpr int LV = (TGC == 16) ? 4 : 3;  // log2 TGC
            const int kc8 = t % NKC, gc = t / NKC;
            const uint8_t* colp = sm.tile + (kc8 / 8) * (kT * 128);
            const int ck = kc8 % 8;
            f2_t acc[4][LV];
            f2_t cur[4];
#pragma unroll
            for (int i = 0; i < TGC; ++i) {
                const int tt = gc * TGC + i;
                const uint4 xr = *reinterpret_cast<const uint4*>(colp + tt * 128 + ((ck ^ (tt & 7)) << 4));
                const float rt = sm.tokv[tt];
                const f2_t RT = f2_pack(rt, rt);
                const __half2* hp = reinterpret_cast<const __half2*>(&xr);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = __half22float2(hp[e]);
                    cur[e] = f2_mul_sep(f2_pack(x.x, x.y), RT, NZ);
                }
#pragma unroll
                for (int l = 0; l < LV; ++l) {
                    if ((i >> l) & 1) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) cur[e] = f2_add(acc[e][l], cur[e]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[e][l] = cur[e];
                        break;
                    }
                }
            }
            // cur: channels 8 kc8 .. 8 kc8 + 7 of the group; into pair order
            // (index 2 (c mod D/2) + c / (D/2)) for the combine below
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float lo, hi;
                f2_unpack(cur[e], lo, hi);
                const int c = 8 * kc8 + 2 * e;
                sm.gpart[gc * D + 2 * (c % (D / 2)) + c / (D / 2)] = lo;
                sm.gpart[gc * D + 2 * ((c + 1) % (D / 2)) + (c + 1) / (D / 2)] = hi;
            }
        } else {
            // a = x * r1, with the rotation's signs when SIGNS
            widen_row<D, SIGNS>(raw, sm, P);
#pragma unroll
            for (int j = 0; j < H2; ++j) P[j] = f2_mul_sep(P[j], R1, NZ);
            before_spill();
            __syncthreads();  // every row has been read from the tile region
            {
                // the rows of a into the transposed buffer
                constexpr int NCH2 = D / 8;  // 16-byte chunks (two pairs) per half row
                char* lo = reinterpret_cast<char*>(sm.red_lo) + (size_t)t * (D / 2) * 4;
                char* hi = reinterpret_cast<char*>(sm.red_hi) + (size_t)t * (D / 2) * 4;
#pragma unroll
                for (int k = 0; k < 2 * NCH2; ++k) {
                    const int pk = (k % NCH2) ^ (t & (NCH2 - 1));
                    *reinterpret_cast<ulonglong2*>((k < NCH2 ? lo : hi) + pk * 16) =
                        make_ulonglong2(P[2 * k], P[2 * k + 1]);
                }
            }
            __syncthreads();
            {
                // block means: thread t sums chunk column kc (pairs 2 kc, 2 kc + 1)
                // over the TG tokens of group g in the pairwise (binary-counter)
                // order; the NG group sums meet in the top levels of the tree
                constexpr int NCH2 = D / 8, NCH = 2 * NCH2, TG = NCH, NG = kT / TG;
                static_assert(NG * D * 4 <= 4096, "group sums fit below the DQ scratch");
                constexpr int LV = (TG == 32) ? 5 : 4;  // log2 TG
                const int kc = t % NCH, g = t / NCH;
                const char* base = reinterpret_cast<const char*>(kc < NCH2 ? sm.red_lo : sm.red_hi) +
                                   (size_t)g * TG * (D / 2) * 4;
                const int kh = kc % NCH2;
                f2_t acc[2][LV];
                f2_t cur[2];
#pragma unroll
                for (int i = 0; i < TG; ++i) {
                    const int tt = g * TG + i;
                    const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(base + (size_t)i * (D / 2) * 4 +
                                                                               ((kh ^ (tt & (NCH2 - 1))) << 4));
                    cur[0] = x.x;
                    cur[1] = x.y;
#pragma unroll
                    for (int l = 0; l < LV; ++l) {
                        if ((i >> l) & 1) {
                            cur[0] = f2_add(acc[0][l], cur[0]);
                            cur[1] = f2_add(acc[1][l], cur[1]);
                        } else {
                            acc[0][l] = cur[0];
                            acc[1][l] = cur[1];
                            break;
                        }
                    }
                }
                // cur: the sum over the group (pair order index 4 kc .. 4 kc + 3)
                *reinterpret_cast<ulonglong2*>(sm.gpart + g * D + 4 * kc) = make_ulonglong2(cur[0], cur[1]);
            }
        }
        __syncthreads();
        if (t < D) {
            // pair-order index t: channel c = pair t >> 1 of half t & 1
            constexpr int NG = kNsnTileMeans ? kT / (D / 8) : kT / (D / 4);
            float gs[NG];
#pragma unroll
            for (int k = 0; k < NG; ++k) gs[k] = sm.gpart[k * D + t];
#pragma unroll
            for (int w = 1; w < NG; w *= 2) {
#pragma unroll
                for (int k = 0; k < NG; k += 2 * w) gs[k] = __fadd_rn(gs[k], gs[k + w]);
            }
            // the mean of the signed rows; the stored mean is of the unsigned
            // ones (a sign flip commutes exactly with the sum and the rounding);
            // the tile holds the unsigned values
            const int c = (t >> 1) + (t & 1) * H2;
            float of = __fmul_rn(gs[0], 1.0f / 128.0f);
            if (kNsnTileMeans && SIGNS && sign16(sm.sgn2, c)) of = -of;
            if constexpr (DQ) {
                sm.vec[t] = of;
                const float m = warp_max_abs(of);
                if ((t & 31) == 0) dqs[8 + (t >> 5)] = m;
            } else {
                const __half o16 = __float2half_rn(of);
                out.off[c] = (SIGNS && sign16(sm.sgn2, c)) ? __hneg(o16) : o16;
                sm.vec[t] = __half2float(o16);
            }
        }
        if constexpr (DQ) {
            // 4-bit o and s1 (double quantization), into the block record
            __syncthreads();
            constexpr float kC = 12582912.0f;  // 1.5 * 2^23: fma(y, 1, kC) = kC + rne(y)
            uint8_t* rec = reinterpret_cast<uint8_t*>(out.off);
            float mo = dqs[8];
#pragma unroll
            for (int w = 1; w < D / 32; ++w) mo = fmaxf(mo, dqs[8 + w]);
            const __half so16 = __float2half_rn(__fdiv_rn(mo, 7.0f));
            const float so = __half2float(so16);
            const float invo = so > 0.0f ? __fdiv_rn(1.0f, so) : 0.0f;
            if (t < D) {
                // e = q + 8, q = clamp(rne(o / sigma_o), -7, 7); the rows carry
                // the signs: o_hat of the signed mean, the code of the unsigned
                const float r = fminf(fmaxf(__fmaf_rn(sm.vec[t], invo, kC + 8.0f), kC + 1.0f), kC + 15.0f);
                const int q = (int)(__float_as_uint(r) & 15u) - 8;
                sm.vec[t] = __fmul_rn((float)q, so);
                const int c = (t >> 1) + (t & 1) * H2;
                dq_e[c] = (uint8_t)(((SIGNS && sign16(sm.sgn2, c)) ? -q : q) + 8);
            }
            float mn = dqs[0], mx = dqs[4];
#pragma unroll
            for (int w = 1; w < 4; ++w) {
                mn = fminf(mn, dqs[w]);
                mx = fmaxf(mx, dqs[4 + w]);
            }
            const __half lo16 = __float2half_rn(mn);
            const float lo = __half2float(lo16);
            const float span = fmaxf(__fsub_rn(mx, lo), 0.0f);
            const __half st16 = __float2half_rn(__fdiv_rn(span, 15.0f));
            const float st = __half2float(st16);
            const float invs = st > 0.0f ? __fdiv_rn(1.0f, st) : 0.0f;
            const float rq = fminf(fmaxf(__fmaf_rn(__fsub_rn(s1, lo), invs, kC), kC), kC + 15.0f);
            const uint32_t qs = __float_as_uint(rq) & 15u;
            const uint32_t qn = __shfl_xor_sync(0xffffffffu, qs, 1);
            if ((t & 1) == 0) rec[D / 2 + t / 2] = (uint8_t)(qs | (qn << 4));
            if (t == 0) {
                __half* pr = reinterpret_cast<__half*>(rec + dq_params_at<D>());
                pr[0] = so16;
                pr[1] = lo16;
                pr[2] = st16;
#pragma unroll
                for (int i = dq_params_at<D>() + 6; i < dq_record_bytes<D>(); ++i) rec[i] = 0;
            }
            __syncthreads();
            if (t < D / 2) rec[t] = (uint8_t)(dq_e[2 * t] | (dq_e[2 * t + 1] << 4));
        }
        __syncthreads();
        after_means();  // the transposed buffer is free again
        if constexpr (kNsnTileMeans) {
            // a = x * r1 (the row leaves its fp16 form only now)
            widen_row<D, SIGNS>(raw, sm, P);
#pragma unroll
            for (int j = 0; j < H2; ++j) P[j] = f2_mul_sep(P[j], R1, NZ);
        }
        // b = a - s (.) o
        const uint32_t mv = smem_u32(sm.vec);
#pragma unroll
        for (int j = 0; j < H2; j += 2) {
            f2_t m0, m1;
            lds_f2x2(mv + 8 * j, m0, m1);
            P[j] = f2_sub(P[j], m0);
            P[j + 1] = f2_sub(P[j + 1], m1);
        }
        const float n2 = __fsqrt_rn(row_sumsq<H2, false>(P, NZ));
        const float s2 = __fmul_rn(n2, rsqd);
        kscale = n2 > 0.0f ? __fdiv_rn(c0, n2) : 0.0f;
        if constexpr (DQ) out.tok[t] = __float2half_rn(s2);
        else reinterpret_cast<__half2*>(out.tok)[t] = __halves2half2(__float2half_rn(s1), __float2half_rn(s2));
    } else if constexpr (MODE == kNsep) {
        widen_row<D, SIGNS>(raw, sm, P);
        const float n = __fsqrt_rn(row_sumsq<H2, true>(P, f2_t(0)));
        out.tok[t] = __float2half_rn(n);
        kscale = n > 0.0f ? __fdiv_rn(c0, n) : 0.0f;
    } else {
        widen_row<D, SIGNS>(raw, sm, P);
        kscale = c0;
    }

    if constexpr (HAD) fwht2<H2>(P);
    if constexpr (MODE != kNaive || HAD) {
        const f2_t K2 = f2_pack(kscale, kscale);
#pragma unroll
        for (int j = 0; j < H2; ++j) P[j] = f2_mul(P[j], K2);
    }

    constexpr float kQ = (float)L::kQmax;
    constexpr float kC = 12582912.0f + (float)L::kOff;  // 1.5 * 2^23 + offset
    if constexpr (MODE == kNaive) {
        __syncthreads();  // every row has been read from the tile the codes are staged over
        // max |x| over the row (exact in any order): eight independent chains
        float mp[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < H2; ++j) {
            float lo, hi;
            f2_unpack(P[j], lo, hi);
            mp[j & 7] = fmaxf(mp[j & 7], fmaxf(fabsf(lo), fabsf(hi)));
        }
        const float m = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                              fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        const __half s16 = __float2half_rn(__fdiv_rn(m, kQ));
        out.tok[t] = s16;
        const float sf = __half2float(s16);
        const float inv = sf > 0.0f ? __fdiv_rn(1.0f, sf) : 0.0f;
        // some |x * inv| of this row rounds past qmax (an fp16 subnormal
        // scale): the exact sign of m * inv - (qmax + 1/2); the warp takes
        // the clamped packer only when one of its rows needs it
        const bool clamp = __fmaf_rn(m, inv, -(kQ + 0.5f)) >= 0.0f;
        uint32_t w[L::kWords];
        if (__any_sync(0xffffffffu, clamp)) codes_from_regs<D, BITS, true, true>(P, nullptr, w, inv);
        else codes_from_regs<D, BITS, false, true>(P, nullptr, w, inv);
        store_codes<D, BITS>(out, t, w);
    } else {
        // per-channel absmax over the block: one redux per channel and warp
        // gives the max over the warp's 32 tokens to every lane; lane k
        // stores the four values of pairs 2k, 2k + 1 (pair order)
        const int lane = t & 31, warp = t >> 5;
        float* wm = sm.gpart + warp * D;
        static_assert(4 * D * 4 <= kGpartBytes, "warp maxima fit the partials buffer");
#pragma unroll
        for (int j = 0; j < H2; j += 2) {
            float a0, b0, a1, b1;
            f2_unpack(P[j], a0, b0);
            f2_unpack(P[j + 1], a1, b1);
            const float r0 = warp_max_abs(a0), r1 = warp_max_abs(b0);
            const float r2 = warp_max_abs(a1), r3 = warp_max_abs(b1);
            if (lane == ((j >> 1) & 31)) *reinterpret_cast<float4*>(wm + 2 * j) = make_float4(r0, r1, r2, r3);
        }
        __syncthreads();
        int clamp = 0;
        if (t < D) {
            // t indexes the pair-order vector: pair t >> 1, lane t & 1
            const int c = (t >> 1) + (t & 1) * H2;
            const float m = fmaxf(fmaxf(sm.gpart[t], sm.gpart[D + t]), fmaxf(sm.gpart[2 * D + t], sm.gpart[3 * D + t]));
            const __half s16 = __float2half_rn(__fdiv_rn(m, kQ));
            out.chan[c] = s16;
            const float sf = __half2float(s16);
            const float inv = sf > 0.0f ? __fdiv_rn(1.0f, sf) : 0.0f;
            sm.vec[t] = inv;
            // some |u * inv| of this channel rounds past qmax (an fp16
            // subnormal scale): the exact sign of m * inv - (qmax + 1/2)
            clamp = __fmaf_rn(m, inv, -(kQ + 0.5f)) >= 0.0f;
        }
        const int any_clamp = __syncthreads_or(clamp);
        uint32_t w[L::kWords];
        if (!any_clamp) codes_from_regs<D, BITS, false>(P, sm.vec, w);
        else codes_from_regs<D, BITS, true>(P, sm.vec, w);
        store_codes<D, BITS>(out, t, w);
    }
}

}  // namespace kvq
