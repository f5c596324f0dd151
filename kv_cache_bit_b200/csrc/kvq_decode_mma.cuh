// kvq_decode_mma.cuh -- decode attention over the packed cache on the tensor
// cores (head dim 128).  Included once, by kvq_api.cu.
//
// Work: a persistent grid.  The quantized blocks of all (batch, kv head)
// pairs are laid end to end and split into equal contiguous ranges, one per
// CTA; warp w of a CTA takes blocks w, w + kNW, ... of the range (so the
// warps of a CTA stream neighbouring blocks) through its own ring of kRing
// shared-memory slots, and writes one partial softmax state per pair segment
// it covers, with the code term already rotated back to the original
// domain.  A slot holds one tensor's half block (packed codes, per-token parameters,
// and on the first half the channel scales and NSN means), brought in by 1-D
// bulk copies (no multicast) that complete on the slot's mbarrier.  Per block
// the unit order is K lo, V lo, K hi, V hi.  decode_combine_mma_kernel then
// merges the partials of each pair with its fp16 residual tokens.
//
// Per block (all G query heads of the kv head at once, G <= 8):
//   scores  S[tok][col] = sum_c code[tok][c] * q'[c][col] with
//           mma.m16n8k16 (A = codes, unpacked from nibbles straight into the
//           fragment registers; B = q' = qt (.) sigma^K scaled by a power of
//           two and split into fp16 hi + lo columns, so the fp32 operand
//           keeps ~22 bits; codes are exact in fp16).
//   softmax logits in the log2 domain, online max/sum per head.
//   values  Acc[c][col] += sum_tok code^V[tok][c] * P'[tok][col] with
//           mma.m16n8k16 (A = V codes transposed: the pair-interleaved V
//           rows give two tokens' codes of a channel per 32-bit word; B =
//           P' = p * nu split into hi + lo, moved from
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
constexpr int kRing = 3;  // slots per warp

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
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

// D += A * B, m16n8k16, fp16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B (the accumulation starts from zero), m16n8k16, fp16 inputs.
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// D = A * B + C with C = (c0, c1) on row g and (c2, c3) on row g + 8.
__device__ __forceinline__ void mma16816_c4(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1, float c0, float c1, float c2, float c3) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

// D = A * B + C with the same C pair (c0, c1) on rows g and g + 8.
__device__ __forceinline__ void mma16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1, float c0, float c1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1));
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 1024.0, 1024.0

__device__ __forceinline__ uint32_t h2c(float v) { return pack_h2(v, v); }

// ---------------------------------------------------------------- code unpacking

// K side.  Thread slot t of a quad owns channels [32t, 32t + 32) of a token
// row and turns them into 16 fp16x2 pairs; pair p holds the codes of
// channels (kc_a(p), kc_b(p)) relative to 32t.
template <int BITS>
struct KUnpack;

// INT4 (kSubnormal): the offset-binary code e = q + kOff of a nibble is
// used in place, as an fp16 subnormal: a nibble at bits 4j .. of a byte,
// masked out of its 16-bit half, reads e * f * 2^-24 with the field scale
// f = 16^j (cscale), one mask per pair of codes and no fp16 arithmetic.  The kernel scales the other operand
// of a channel by 1/f, folds 2^24 into the scales it applies to the fp32
// results, and removes the bias kOff times the sum of the other operand: for
// the scores with one MMA chain per block against a constant A of
// -kOff f 2^-24 per channel, for the values from the unit's sum of P' as
// the value chains' starting C.  Subnormal fp16 inputs are exact values; the
// tensor core's sum of such products measured within 2^-19 of the sum of
// their magnitudes (against 2^-23 for normal inputs), which the bias
// (|e| <= 2 qmax + 1 against |q| <= qmax) costs about one bit of.
constexpr float kTwo24 = 16777216.0f;  // 2^24

// fp16x2 bits of -kOff * f * 2^-24 (both halves); kOff * f < 1024 keeps it subnormal
__host__ __device__ constexpr uint32_t sub_bias_h2(int off_times_f) {
    return (0x8000u | (uint32_t)off_times_f) * 0x00010001u;
}

template <>
struct KUnpack<4> {
    static constexpr int kPairGroup = 4;  // pairs 4i + j: channels 8i + j and 8i + 4 + j
    static constexpr bool kSubnormal = true;
    static constexpr int kOff = 8;
    // field scale of channel c (low nibble 1, high nibble 16)
    __host__ __device__ static constexpr int cscale(int c) { return (c & 1) ? 16 : 1; }
    __device__ static int ca(int p) { return 8 * (p >> 2) + (p & 3); }
    __device__ static int cb(int p) { return ca(p) + 4; }
    // row points at the row's first byte; even pairs p hold e * 2^-24, odd
    // pairs (high nibbles) 16 e * 2^-24
    __device__ static void run(const uint8_t* row, int t, uint32_t (&pr)[16]) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * t);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t W = w[i], W8 = w[i] >> 8;
            pr[4 * i + 0] = W & 0x000F000Fu;
            pr[4 * i + 1] = W & 0x00F000F0u;
            pr[4 * i + 2] = W8 & 0x000F000Fu;
            pr[4 * i + 3] = W8 & 0x00F000F0u;
        }
    }
};

// 2-bit fields j = 0..3 of a byte pair: value 1024 + e * 4^j, q = e - off.
// (INT2 codes are converted to exact q: as subnormals with field scales up
// to 64 the score and value sums measured about four times the error of
// this form.)
template <int OFF>
__device__ __forceinline__ uint32_t dec2(uint32_t x, int j) {
    const float m = float(1 << (2 * j));
    return h2_fma(lop_and_or(x, 0x00030003u << (2 * j), kMagic), h2c(1.0f / m), h2c(-(1024.0f / m + OFF)));
}

template <>
struct KUnpack<2> {
    static constexpr bool kSubnormal = false;
    static constexpr int kOff = 0;
    __host__ __device__ static constexpr int cscale(int) { return 1; }
    static constexpr int kPairGroup = 8;  // pairs 8i + j: channels 16i + j and 16i + 8 + j
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

// INT3: the 2-bit field of field index jj (bits 2jj, 2jj + 1 of each half)
// and the high bit moved to bit 2jj + 2 form e * 4^jj in the mantissa of
// 1024 + e * 4^jj (two LOP3s); one FMA gives e - 4.
__device__ __forceinline__ uint32_t lop_or_and(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xF8;" : "=r"(r) : "r"(a), "r"(b), "r"(c));  // a | (b & c)
    return r;
}

// x: 2-bit fields at bits 2jj (+16); hs: high bits already at bit 2jj + 2 (+16)
__device__ __forceinline__ uint32_t dec3(uint32_t x, uint32_t hs, int jj) {
    const float m = float(1 << (2 * jj));
    const uint32_t u = lop_and_or(x, 0x00030003u << (2 * jj), kMagic);
    const uint32_t v = lop_or_and(u, hs, 0x00040004u << (2 * jj));
    return h2_fma(v, h2c(1.0f / m), h2c(-(1024.0f / m + 4.0f)));
}

// shift moving bit j to bit 2 (j & 3) + 2
__device__ __forceinline__ uint32_t hi_to(uint32_t h, int j) {
    const int sh = 2 * (j & 3) + 2 - j;
    return sh >= 0 ? (h << sh) : (h >> (-sh));
}

template <>
struct KUnpack<3> {
    static constexpr bool kSubnormal = false;
    static constexpr int kOff = 0;
    __host__ __device__ static constexpr int cscale(int) { return 1; }
    static constexpr int kPairGroup = 8;  // pairs 8i + j: channels 16i + j and 16i + 8 + j
    __device__ static int ca(int p) { return 16 * (p >> 3) + (p & 7); }
    __device__ static int cb(int p) { return ca(p) + 8; }
    __device__ static void run(const uint8_t* row, int t, uint32_t (&pr)[16]) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * t);
        const uint32_t H = *reinterpret_cast<const uint32_t*>(row + 32 + 4 * t);
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            // high bits of channels 16i + j and 16i + 8 + j at bits j and 16 + j
            const uint32_t Hi = prmt(H, 0u, i ? 0x4342u : 0x4140u);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                pr[8 * i + j] = dec3(j < 4 ? w[i] : (w[i] >> 8), hi_to(Hi, j), j & 3);
        }
    }
};

// V side.  Thread g of a warp owns channels [16g, 16g + 16) of a token row.
// V rows are stored pair-interleaved (word u of the pair block of tokens 2k,
// 2k + 1 holds unit u of both rows, see pairv_layout), so the registers the
// value MMA wants, (code[2k][c], code[2k + 1][c]) for c = 16g + j, come
// straight from the pair block pb: pr[j] for j = 0..15.
template <int BITS>
struct VUnpack;

template <>
struct VUnpack<4> {
    static constexpr bool kSubnormal = true;  // e * 2^-24; odd channels (high nibbles) 16 e * 2^-24
    static constexpr int kOff = 8;
    // field scale of register i of run() (the MMA's row g for even i, g + 8 for odd)
    __host__ __device__ static constexpr int vscale(int i) { return (i & 1) ? 16 : 1; }
    // units 4g .. 4g + 3: the 16-byte chunk g, at g ^ (2 (k & 1))
    __device__ static void run(const uint8_t* pb, int k, int g, uint32_t (&pr)[16]) {
        const uint4 v = *reinterpret_cast<const uint4*>(pb + 16 * (g ^ pairv_chunk_xor<4>(k)));
        const uint32_t x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // unit 4g + i of both rows: channels 16g + 4i .. + 3
            const uint32_t x = x4[i], x8 = x >> 8;
            pr[4 * i + 0] = x & 0x000F000Fu;
            pr[4 * i + 1] = x & 0x00F000F0u;
            pr[4 * i + 2] = x8 & 0x000F000Fu;
            pr[4 * i + 3] = x8 & 0x00F000F0u;
        }
    }
};

template <>
struct VUnpack<2> {
    static constexpr bool kSubnormal = false;
    static constexpr int kOff = 0;
    __host__ __device__ static constexpr int vscale(int) { return 1; }
    // units 2g, 2g + 1: words 2g, 2g + 1 of the pair block
    __device__ static void run(const uint8_t* pb, int, int g, uint32_t (&pr)[16]) {
        const uint2 v = *reinterpret_cast<const uint2*>(pb + 8 * g);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t x = hh ? v.y : v.x;  // channels 16g + 8hh .. + 7
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
    static constexpr bool kSubnormal = false;
    static constexpr int kOff = 0;
    __host__ __device__ static constexpr int vscale(int) { return 1; }
    // 2-bit plane: units 2g, 2g + 1 (words 2g, 2g + 1); bit plane: unit 16 + g
    __device__ static void run(const uint8_t* pb, int, int g, uint32_t (&pr)[16]) {
        const uint2 v = *reinterpret_cast<const uint2*>(pb + 8 * g);
        // bit j: channel 16g + j of row 2k; bit 16 + j: of row 2k + 1
        const uint32_t hh2 = *reinterpret_cast<const uint32_t*>(pb + 64 + 4 * g);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t x = hh ? v.y : v.x;
            const uint32_t hsrc = hh ? (hh2 >> 8) : hh2;  // channel 8hh + j at bits j, 16 + j
#pragma unroll
            for (int j = 0; j < 8; ++j)
                pr[8 * hh + j] = dec3(j < 4 ? x : (x >> 8), hi_to(hsrc, j), j & 3);
        }
    }
};

// ---------------------------------------------------------------- slot layout

constexpr int kUT = 64;  // tokens per staging unit (half a block)
constexpr int kMaxCtasPerSM = 4;  // cap of the persistent grid: this many CTAs per SM

// A unit is one tensor's half block: packed codes and per-token parameters of
// 64 tokens; the first half also carries the block's channel scales and NSN
// channel means.
//
// Under DQ the block record (codes of o and s1, their fp16 parameters) sits
// between the token parameters and the channel scales, and both halves
// carry it (each half's tokens need their s1 codes).
template <int D, int BITS, int MODE>
struct SlotLayout {
    static constexpr bool kDq = MODE == kNsnDq;
    static constexpr int kRB = D * BITS / 8;
    static constexpr int kNtok = tok_params(MODE);
    static constexpr int kCodes = 0;
    static constexpr int kTok = kUT * kRB;
    static constexpr int kRec = kTok + kUT * kNtok * 2;  // DQ record
    static constexpr int kChan = kRec + (kDq ? dq_record_bytes<D>() : 0);
    static constexpr int kOff = kChan + ((MODE != kNaive) ? D * 2 : 0);
    static constexpr int kBytesLo = kOff + ((MODE == kNsn) ? D * 2 : 0);  // first half
    static constexpr int kBytesHi = kChan;                                 // second half
    // DQ: s1 of the unit's 64 tokens as fp32, rebuilt from the record by the
    // warp once the unit has landed (not a copy target)
    static constexpr int kS1 = (kBytesLo + 15) / 16 * 16;
    static constexpr int kStride = (kS1 + (kDq ? kUT * 4 : 0) + 127) / 128 * 128;
    static_assert(kRec % 16 == 0 && kChan % 16 == 0, "bulk copies start on 16-byte boundaries");
};

// The codes of o for 16 channels (8 bytes at p) as exact fp16 pairs q = e - 8
// (channels 2k, 2k + 1 in pair k).
__device__ __forceinline__ void dq_o_pairs(const uint8_t* p, __half2 (&o)[8]) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t b = ((k < 4 ? w.x : w.y) >> (8 * (k & 3))) & 0xFFu;
        o[k] = __floats2half2_rn((float)((int)(b & 15u) - 8), (float)((int)(b >> 4) - 8));
    }
}

// DQ: s1 of the unit's 64 tokens (half `half` of the block) rebuilt from the
// slot's record into the slot's fp32 s1 area, two tokens per lane.
template <int D, typename SL>
__device__ __forceinline__ void dq_fill_s1(uint8_t* slot, int half, int lane) {
    float* s1 = reinterpret_cast<float*>(slot + SL::kS1);
    s1[2 * lane] = dq_s1<D>(slot + SL::kRec, 64 * half + 2 * lane);
    s1[2 * lane + 1] = dq_s1<D>(slot + SL::kRec, 64 * half + 2 * lane + 1);
    __syncwarp();
}

// Rotated-query table (fp32): channel c of head j at j * kQS + c + 4 (c / 32).
// The B-fragment build reads 16-byte chunks of the 32-channel slice t of one
// head per thread quad; the 4-word skew per slice puts the four slices of a
// quarter warp on different banks.
constexpr int kQS = 128 + 16;
__host__ __device__ constexpr int qs_index(int j, int c) { return j * kQS + c + 4 * (c >> 5); }
// Raw-query table (fp16, exact copies of the query): channels (c, c + 1),
// c even, of head j in 32-bit word j * kQWW + c / 2 + c / 64.  The NSN offset
// dot product reads the words of channels 16g + 2k of head t across a warp;
// the row stride (2 mod 32 words) and the one-word skew per 64 channels put
// the 32 lanes on 32 different banks.
constexpr int kQWW = 64 + 2;
__host__ __device__ constexpr int qw_word(int j, int c) { return j * kQWW + (c >> 1) + (c >> 6); }

// Partial record of one (segment, head): [m, l, 0, 0, acc[D]] with acc in the
// original domain (the code term already rotated back, plus the NSN offset
// term); the two pad floats keep acc 16-byte aligned for vector stores.
template <int D>
__host__ __device__ constexpr int part_stride() { return 4 + D; }

template <int D, int BITS, int MODE, int GP>
struct MmaSmem {
    static constexpr int kRing0 = 0;
    static constexpr int kBars = kNW * kRing * SlotLayout<D, BITS, MODE>::kStride;
    static constexpr int kQ = kBars + kNW * kRing * 8;        // per warp: raw q [GP][kQWW] fp16 pairs
    static constexpr int kQs = kQ + kNW * GP * kQWW * 4;      // per warp: skewed scaled rotated q [GP][kQS]
    static constexpr int kQsc = kQs + kNW * GP * kQS * 4;     // per warp: [GP] scales
    static constexpr int kBytes = kQsc + kNW * GP * 4 + 128;
};

template <int D, int BITS, int MODE, int GP>
__host__ __device__ constexpr int mma_smem_bytes() {
    return MmaSmem<D, BITS, MODE, GP>::kBytes;
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Split of `work` blocks over nctas CTAs: the first r CTAs take q + 1 blocks,
// the others q (q = work / nctas, r = work % nctas; work < 2^31).
struct CtaSplit {
    int q, r;
    __host__ __device__ CtaSplit(long long work, long long nctas)
        : q((int)(work / nctas)), r((int)(work % nctas)) {}
    __host__ __device__ int start(int c) const { return c * q + min(c, r); }
    // CTA holding block x
    __host__ __device__ int cta_of(int x) const {
        const int big = r * (q + 1);
        return x < big ? x / (q + 1) : r + (x - big) / q;
    }
};

// Partial slot of warp w of CTA c for pair p: CTA ranges are contiguous and
// ordered, so c + p is unique per (CTA, pair) that meet; slots < kNW * (nctas + pairs).
__host__ __device__ __forceinline__ long long part_slot(long long c, int w, long long p) {
    return (c + p) * kNW + w;
}

// ---------------------------------------------------------------- the kernel

__device__ __forceinline__ uint32_t cvt_h2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// fp32 x -> (hi, lo) fp16 pair with hi = fp16(x), lo = fp16(x - hi); packed
// with hi in the low half.
__device__ __forceinline__ uint32_t split_h2(float x) {
    const __half h = __float2half_rn(x);
    return cvt_h2(__half2float(h), x - __half2float(h));
}

// Column layout of every n-tile (8 columns): column 2j + part holds part
// (0 = hi, 1 = lo) of head 4n + j.  Thread (g, t) of a warp therefore owns
// head 4n + t of every n-tile in the C fragments and sums its two columns.
// Partial state of a (warp, pair) segment goes to slot part_slot() of a.part:
// [m (log2 units), l, pad, pad, acc[D] (original domain)] per head
// (part_stride floats).
// The NSN and INT3 instantiations with one n-tile of query heads are held to
// three resident CTAs per SM (168 registers), where the register allocator
// otherwise spills or settles for fewer CTAs; the others are left to it.
template <int D, int BITS, int MODE, bool HAD, int GP>
__global__ void __launch_bounds__(kNW * 32, ((BITS == 3 || is_nsn(MODE)) && GP == 4) ? 3 : 0)
    decode_mma_kernel(DecodeArgs a) {
    static_assert(D == 128, "tensor-core decode is built for head dim 128");
    using SL = SlotLayout<D, BITS, MODE>;
    using SM = MmaSmem<D, BITS, MODE, GP>;
    constexpr int NT = GP / 4;  // n-tiles (heads per thread)
    constexpr bool PCH = MODE != kNaive;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    constexpr float kTau = 8.0f;  // reference-max slack (log2 units): p <= 2^kTau
    using KU = KUnpack<BITS>;
    using VU = VUnpack<BITS>;
    constexpr bool KB = KU::kSubnormal, VB = VU::kSubnormal;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int G = a.G;
    const int nbq = a.nbq;
    const int nb_cap = a.cap / kT;
    const int cta = blockIdx.x;
    const CtaSplit split(a.work, a.nwarps / kNW);
    const int c0 = split.start(cta), c1 = split.start(cta + 1);
    const int w0 = c0 + warp;  // this warp's blocks: w0, w0 + kNW, ... < c1
    const int nmine = w0 < c1 ? (c1 - w0 + kNW - 1) / kNW : 0;
    const int nunits = 4 * nmine;

    uint8_t* my_ring = smem_raw + SM::kRing0 + warp * kRing * SL::kStride;
    uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem_raw + SM::kBars) + warp * kRing;
    uint32_t* wqw = reinterpret_cast<uint32_t*>(smem_raw + SM::kQ) + warp * GP * kQWW;  // [GP][kQWW], qw_word
    float* wqs = reinterpret_cast<float*>(smem_raw + SM::kQs) + warp * GP * kQS;    // [GP][kQS]
    float* wqsc = reinterpret_cast<float*>(smem_raw + SM::kQsc) + warp * GP;        // [GP]

    if (lane < kRing) mbar_init(&my_bars[lane], 1);
    fence_mbar_init();
    __syncwarp();

    // The units are issued strictly in order; the block of the next unit to
    // issue is kept as a (pair, block) cursor instead of dividing per unit.
    int iss_pair = nmine > 0 ? w0 / nbq : 0;
    int iss_blk = nmine > 0 ? w0 - iss_pair * nbq : 0;
    auto issue = [&](int u) {
        const int pair = iss_pair, blk = iss_blk;
        const int ten = u & 1;
        const int half = (u >> 1) & 1;
        uint8_t* slot = my_ring + (u % kRing) * SL::kStride;
        uint64_t* bar = &my_bars[u % kRing];
        const size_t row0 = (size_t)pair * a.cap + (size_t)blk * kT + (size_t)half * kUT;
        const size_t bi = ((size_t)pair * nb_cap + blk) * D;
        mbar_expect_tx(bar, half ? SL::kBytesHi : SL::kBytesLo);
        bulk_load(slot + SL::kCodes, (ten ? a.codes[1] : a.codes[0]) + row0 * SL::kRB, kUT * SL::kRB, bar);
        bulk_load(slot + SL::kTok, (ten ? a.tok[1] : a.tok[0]) + row0 * SL::kNtok, kUT * SL::kNtok * 2, bar);
        if (SL::kDq)
            bulk_load(slot + SL::kRec, (ten ? a.off[1] : a.off[0]) + ((size_t)pair * nb_cap + blk) * off_words<D, MODE>(),
                      dq_record_bytes<D>(), bar);
        if (!half) {
            if (PCH) bulk_load(slot + SL::kChan, (ten ? a.chan[1] : a.chan[0]) + bi, D * 2, bar);
            if (MODE == kNsn) bulk_load(slot + SL::kOff, (ten ? a.off[1] : a.off[0]) + bi, D * 2, bar);
        }
    };
    // advance the cursor past unit u (every lane keeps the same cursor)
    auto advance = [&](int u) {
        if ((u & 3) == 3) {
            iss_blk += kNW;
            while (iss_blk >= nbq) { iss_blk -= nbq; ++iss_pair; }
        }
    };
    // the kernel is a programmatic dependent of the one ahead of it (an
    // append, or the previous call's combine): nothing of the cache, the
    // queries or the workspace is touched before that one has finished; the
    // combine kernel behind this one may be scheduled from here on
    grid_dep_wait();
    grid_dep_launch();
    int issued = min(kRing, nunits);
    for (int u = 0; u < issued; ++u) {
        if (lane == 0) issue(u);
        advance(u);
    }
    int waited = 0;
    bool ok = true;
    auto wait_unit = [&](int u) -> bool {
        if (!mbar_wait(&my_bars[u % kRing], (u / kRing) & 1, KVQ_WAIT_LIMIT(1u << 26))) return false;
        waited = u + 1;
        return true;
    };
    // unit u consumed: its slot takes unit u + kRing
    auto release = [&](int u) {
        __syncwarp();
        if (u + kRing < nunits) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(u + kRing);
            }
            advance(u + kRing);
            issued = u + kRing + 1;
        }
    };

    const float alpha2 = a.scale * kLog2e;
    const bool blo = (g & 1) != 0;  // B column of this thread: head 4n + g/2, part g%2
    const int tr0 = g, tr1 = 8 + g;  // tokens of the score fragment rows (and of P' rows)

    int pos = 0;
    while (pos < nmine && ok) {
        const int x0 = w0 + pos * kNW;
        const int pair = x0 / nbq;
        // blocks of this warp inside the pair: x0, x0 + kNW, ... < (pair + 1) * nbq
        const int seg = min(nmine - pos, ((pair + 1) * nbq - x0 + kNW - 1) / kNW);
        const int b = pair / a.H, h = pair % a.H;
        // ---- segment prologue: this pair's queries, rotated and scaled (lane owns 4 channels)
#pragma unroll
        for (int j = 0; j < GP; ++j) {
            const uint2 raw = (j < G) ? *reinterpret_cast<const uint2*>(
                                            a.q + ((size_t)b * a.H * G + (size_t)h * G + j) * D + 4 * lane)
                                      : make_uint2(0u, 0u);
            wqw[qw_word(j, 4 * lane)] = raw.x;
            wqw[qw_word(j, 4 * lane + 2)] = raw.y;
            const float2 q01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 q23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            float v[4] = {q01.x, q01.y, q23.x, q23.y};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c = 4 * lane + k;
                if (HAD && a.signs != nullptr && a.signs[c] < 0) v[k] = -v[k];
            }
            if constexpr (HAD) {
                const float x0_ = v[0] + v[1], x1_ = v[0] - v[1], x2_ = v[2] + v[3], x3_ = v[2] - v[3];
                v[0] = x0_ + x2_; v[2] = x0_ - x2_; v[1] = x1_ + x3_; v[3] = x1_ - x3_;
#pragma unroll
                for (int m = 1; m < 32; m <<= 1) {
                    const bool upper = (lane & m) != 0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float o = __shfl_xor_sync(0xffffffffu, v[k], m);
                        v[k] = upper ? (o - v[k]) : (v[k] + o);
                    }
                }
            }
            float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
            for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            // |q'| <= amax * max(sigma) <= amax / qmax (1 + 2^-10): keep it below 2^13
            const float bound = PCH ? amax * (1.001f / (float)QMAX) : amax;
            const float qsc = bound > 0.0f ? pow2i(13 - ceil_log2(bound)) : 1.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                // channels of field scale f meet codes e f 2^-24: 1/f
                const float bs = KB ? 1.0f / (float)KU::cscale(k) : 1.0f;
                wqs[qs_index(j, 4 * lane + k)] = v[k] * qsc * bs;
            }
            if (lane == 0) wqsc[j] = qsc;
        }
        __syncwarp();

        // ---- per-thread state of the segment: heads 4n + t, channels [16g, 16g + 16)
        float m_ref[NT], l_run[NT], kcol[NT];
        float acc[NT][16], acco[NT][16];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            m_ref[n] = -INFINITY;
            l_run[n] = 0.0f;
            // 2^-qsc with the softmax scale (log2 units) and the fixed token
            // factor of the mode folded in
            kcol[n] = alpha2 * ((is_nsn(MODE) && !HAD) ? a.sqd : (MODE == kNsep && HAD) ? a.rsqd : 1.0f) /
                      wqsc[4 * n + t] * (KB ? kTwo24 : 1.0f);
#pragma unroll
            for (int k = 0; k < 16; ++k) { acc[n][k] = 0.0f; acco[n][k] = 0.0f; }
        }
        uint32_t bq[NT][16];
        float kb[NT][2];  // -1152 * sum of B over the biased pairs (hi, lo columns)
        float qoK[NT];
        __half2 sigv[8], offv[8];
        float osv = 1.0f;  // DQ: sigma_o of the block's V means

        for (int it = pos; it < pos + seg; ++it) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int uk = 4 * it + 2 * half, uv = uk + 1;
                if (!wait_unit(uk)) { ok = false; break; }
                uint8_t* sk = my_ring + (uk % kRing) * SL::kStride;
                if constexpr (SL::kDq) dq_fill_s1<D, SL>(sk, half, lane);
                if (half == 0) {
                    // B fragments: q' = qs * sigma^K as (hi, lo) fp16 parts; a
                    // group of PG pairs takes 2 PG channels of the slice
                    constexpr int PG = KUnpack<BITS>::kPairGroup;
                    const uint4* sg4 = reinterpret_cast<const uint4*>(sk + SL::kChan) + 4 * t;  // slice t
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const float4* q4 = reinterpret_cast<const float4*>(&wqs[qs_index(4 * n + (g >> 1), 32 * t)]);
#pragma unroll
                        for (int grp = 0; grp < 16 / PG; ++grp) {
                            float qv[2 * PG], sv[2 * PG];
#pragma unroll
                            for (int v = 0; v < PG / 2; ++v) {
                                const float4 f = q4[grp * (PG / 2) + v];
                                qv[4 * v] = f.x; qv[4 * v + 1] = f.y; qv[4 * v + 2] = f.z; qv[4 * v + 3] = f.w;
                            }
#pragma unroll
                            for (int v = 0; v < PG / 4; ++v) {
                                const uint4 hv = PCH ? sg4[grp * (PG / 4) + v] : make_uint4(0u, 0u, 0u, 0u);
                                const uint32_t w4[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                                for (int w = 0; w < 4; ++w) {
                                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[w]));
                                    sv[8 * v + 2 * w] = PCH ? f.x : 1.0f;
                                    sv[8 * v + 2 * w + 1] = PCH ? f.y : 1.0f;
                                }
                            }
#pragma unroll
                            for (int j = 0; j < PG; ++j) {
                                const int p = PG * grp + j;
                                const float fa = qv[j] * sv[j];            // channel ca(p)
                                const float fb = qv[PG + j] * sv[PG + j];  // channel cb(p)
                                const __half2 hh = __floats2half2_rn(fa, fb);
                                if (blo) {
                                    const float2 hf = __half22float2(hh);
                                    bq[n][p] = cvt_h2(fa - hf.x, fb - hf.y);
                                } else {
                                    bq[n][p] = *reinterpret_cast<const uint32_t*>(&hh);
                                }
                            }
                        }
                    }
                    if constexpr (KB) {
                        // bias of the score chains: A = -kOff f 2^-24 for the
                        // field scale f of each pair's channels (a0, a1: pair
                        // 2s of k-step s; a2, a3: pair 2s + 1), whose B carries
                        // 1/f; pairs p and p + 4 have the scale of channel p & 3
                        constexpr uint32_t z0 = sub_bias_h2(KU::kOff * KU::cscale(0));
                        constexpr uint32_t z1 = sub_bias_h2(KU::kOff * KU::cscale(1));
                        constexpr uint32_t z2 = sub_bias_h2(KU::kOff * KU::cscale(2));
                        constexpr uint32_t z3 = sub_bias_h2(KU::kOff * KU::cscale(3));
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            float c0[4], c1[4];
                            mma16816_z(c0, z0, z0, z1, z1, bq[n][0], bq[n][1]);
                            mma16816_z(c1, z2, z2, z3, z3, bq[n][2], bq[n][3]);
#pragma unroll
                            for (int s = 2; s < 8; s += 2) {
                                mma16816(c0, z0, z0, z1, z1, bq[n][2 * s], bq[n][2 * s + 1]);
                                mma16816(c1, z2, z2, z3, z3, bq[n][2 * s + 2], bq[n][2 * s + 3]);
                            }
                            kb[n][0] = c0[0] + c1[0];
                            kb[n][1] = c0[1] + c1[1];
                        }
                    }
                    if constexpr (is_nsn(MODE)) {
                        // q . o^K for head 4n + t: lanes (g) split the channels;
                        // under DQ o = (e - 8) sigma_o, with sigma_o applied once
                        __half2 okv[8];
                        float osc = 1.0f;
                        if constexpr (MODE == kNsn) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) okv[k] = reinterpret_cast<const __half2*>(sk + SL::kOff)[8 * g + k];
                        } else {
                            dq_o_pairs(sk + SL::kRec + 8 * g, okv);
                            osc = __half2float(reinterpret_cast<const __half*>(sk + SL::kRec + dq_params_at<D>())[0]);
                        }
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint32_t* qh = &wqw[qw_word(4 * n + t, 16 * g)];  // channels 16g .. 16g + 15
                            float s = 0.0f;
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const float2 o2 = __half22float2(okv[k]);
                                const float2 q2 = __half22float2(*reinterpret_cast<const __half2*>(&qh[k]));
                                s += q2.x * o2.x + q2.y * o2.y;
                            }
#pragma unroll
                            for (int o = 4; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                            qoK[n] = s * (osc * alpha2);
                        }
                    }
                }
                if (!wait_unit(uv)) { ok = false; break; }
                uint8_t* sv = my_ring + (uv % kRing) * SL::kStride;
                if constexpr (SL::kDq) dq_fill_s1<D, SL>(sv, half, lane);
                if (half == 0) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        sigv[k] = PCH ? reinterpret_cast<const __half2*>(sv + SL::kChan)[8 * g + k]
                                      : __floats2half2_rn(1.f, 1.f);
                        offv[k] = (MODE == kNsn) ? reinterpret_cast<const __half2*>(sv + SL::kOff)[8 * g + k]
                                                 : __floats2half2_rn(0.f, 0.f);
                    }
                    // DQ: the codes q of o^V as exact fp16 pairs; sigma_o^V
                    // multiplies the offset term once per unit
                    if constexpr (MODE == kNsnDq) {
                        dq_o_pairs(sv + SL::kRec + 8 * g, offv);
                        osv = __half2float(reinterpret_cast<const __half*>(sv + SL::kRec + dq_params_at<D>())[0]);
                    }
                }
                const __half* tk = reinterpret_cast<const __half*>(sk + SL::kTok);
                const __half* tv = reinterpret_cast<const __half*>(sv + SL::kTok);
                // power-of-two scale keeping p * nu * 2^f <= 2^13 in fp16 (p <= 2^kTau)
                float numax = 0.0f;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int tok = 2 * lane + k;
                    float v;
                    if constexpr (MODE == kNsn) {
                        const float2 s12 = __half22float2(reinterpret_cast<const __half2*>(tv)[tok]);
                        v = s12.x * s12.y * (HAD ? 1.0f : a.sqd);
                    } else if constexpr (MODE == kNsnDq) {
                        v = reinterpret_cast<const float*>(sv + SL::kS1)[tok] * __half2float(tv[tok]) * (HAD ? 1.0f : a.sqd);
                    } else {
                        v = __half2float(tv[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                    }
                    numax = fmaxf(numax, v);
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) numax = fmaxf(numax, __shfl_xor_sync(0xffffffffu, numax, o));
                const int fexp = numax > 0.0f ? 13 - (int)kTau - ceil_log2(numax) : 0;
                const float pscale = pow2i(fexp), pinv = pow2i(-fexp);
                // 2^f with the fixed token factor of the mode
                const float pscale_m =
                    pscale * ((is_nsn(MODE) && !HAD) ? a.sqd : (MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                // ---- scores of the unit's 64 tokens (four independent 16-token tiles)
                float l2[4][NT][2];
                bool over = false;
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    uint32_t pa[16], pb[16];
                    KUnpack<BITS>::run(sk + SL::kCodes + (16 * m4 + tr0) * SL::kRB, t, pa);
                    KUnpack<BITS>::run(sk + SL::kCodes + (16 * m4 + tr1) * SL::kRB, t, pb);
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float d0[4], d1[4];
                        if constexpr (KB)
                            mma16816_c(d0, pa[0], pb[0], pa[1], pb[1], bq[n][0], bq[n][1], kb[n][0], kb[n][1]);
                        else
                            mma16816_z(d0, pa[0], pb[0], pa[1], pb[1], bq[n][0], bq[n][1]);
                        mma16816_z(d1, pa[2], pb[2], pa[3], pb[3], bq[n][2], bq[n][3]);
#pragma unroll
                        for (int s = 2; s < 8; s += 2) {
                            mma16816(d0, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], bq[n][2 * s],
                                     bq[n][2 * s + 1]);
                            mma16816(d1, pa[2 * s + 2], pb[2 * s + 2], pa[2 * s + 3], pb[2 * s + 3],
                                     bq[n][2 * s + 2], bq[n][2 * s + 3]);
                        }
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int tok = 16 * m4 + (r ? tr1 : tr0);
                            const float sv_ = (d0[2 * r] + d0[2 * r + 1]) + (d1[2 * r] + d1[2 * r + 1]);
                            // logit in log2 units: kap (sv q'.k + q.o) alpha2 for NSN
                            if constexpr (MODE == kNsn) {
                                const float2 s12 = __half22float2(reinterpret_cast<const __half2*>(tk)[tok]);
                                l2[m4][n][r] = s12.x * fmaf(sv_, s12.y * kcol[n], qoK[n]);
                            } else if constexpr (MODE == kNsnDq) {
                                const float s1 = reinterpret_cast<const float*>(sk + SL::kS1)[tok];
                                l2[m4][n][r] = s1 * fmaf(sv_, __half2float(tk[tok]) * kcol[n], qoK[n]);
                            } else {
                                l2[m4][n][r] = sv_ * (__half2float(tk[tok]) * kcol[n]);
                            }
                            over |= l2[m4][n][r] > m_ref[n] + kTau;
                        }
                    }
                }
                release(uk);
                // ---- rare: move the reference max up to the unit's max and rescale
                if (__any_sync(0xffffffffu, over)) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float mx = l2[0][n][0];
#pragma unroll
                        for (int m4 = 0; m4 < 4; ++m4) mx = fmaxf(mx, fmaxf(l2[m4][n][0], l2[m4][n][1]));
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        const float mn = fmaxf(m_ref[n], mx);
                        const float corr = fast_exp2(m_ref[n] - mn);
                        m_ref[n] = mn;
                        l_run[n] *= corr;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            acc[n][k] *= corr;
                            if (is_nsn(MODE)) acco[n][k] *= corr;
                        }
                    }
                }
                // ---- P' = p * nu (scaled) and the values, tile by tile
                float dv[NT][8][4];  // set by the first tile's MMAs
                float psum[NT];  // this thread's rows of the unit's sum of P' (biased V codes)
                float lsum[NT], bsum[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) { lsum[n] = 0.0f; bsum[n] = 0.0f; psum[n] = 0.0f; }
                uint32_t bpa[4][NT][2];
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int tok = 16 * m4 + (r ? tr1 : tr0);
                        float nu, s1o = 0.0f;  // nu: the token's value scale times 2^f
                        if constexpr (MODE == kNsn) {
                            const float2 s12 = __half22float2(reinterpret_cast<const __half2*>(tv)[tok]);
                            s1o = s12.x;
                            nu = s12.x * (s12.y * pscale_m);
                        } else if constexpr (MODE == kNsnDq) {
                            s1o = reinterpret_cast<const float*>(sv + SL::kS1)[tok];
                            nu = s1o * (__half2float(tv[tok]) * pscale_m);
                        } else {
                            nu = __half2float(tv[tok]) * pscale_m;
                        }
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const float p = fast_exp2(l2[m4][n][r] - m_ref[n]);
                            lsum[n] += p;
                            if constexpr (is_nsn(MODE)) bsum[n] += p * s1o;
                            const float x_ = p * nu;
                            if constexpr (VB) psum[n] += x_;
                            bpa[m4][n][r] = movmatrix_t(split_h2(x_));
                        }
                    }
                }
                // subnormal codes: the bias (kOff per code, times the field
                // scale of the row) enters the value chains as their starting
                // C, from the unit's sum of P'
                float vlo[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    if constexpr (VB) {
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) psum[n] += __shfl_xor_sync(0xffffffffu, psum[n], o);
                    }
                    vlo[n] = VB ? (-(float)VU::kOff / kTwo24) * psum[n] : 0.0f;  // times the field scale
                }
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    const uint32_t (&bp)[NT][2] = bpa[m4];
                    uint32_t va[16], vb[16];
                    const uint8_t* vbase = sv + SL::kCodes + (16 * m4) * SL::kRB;
                    // k-steps 2t, 2t + 1 of the value MMA: tokens 2t, 2t + 1 (pair t of
                    // the tile) for va and 8 + 2t, 9 + 2t (pair 4 + t) for vb
                    VUnpack<BITS>::run(vbase + t * 2 * SL::kRB, t, g, va);
                    VUnpack<BITS>::run(vbase + (4 + t) * 2 * SL::kRB, t, g, vb);
#pragma unroll
                    for (int tc = 0; tc < 8; ++tc) {
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            if (m4 == 0 && VB)
                                mma16816_c4(dv[n][tc], va[2 * tc], va[2 * tc + 1], vb[2 * tc], vb[2 * tc + 1],
                                            bp[n][0], bp[n][1], (float)VU::vscale(2 * tc) * vlo[n], 0.0f,
                                            (float)VU::vscale(2 * tc + 1) * vlo[n], 0.0f);
                            else if (m4 == 0)
                                mma16816_z(dv[n][tc], va[2 * tc], va[2 * tc + 1], vb[2 * tc], vb[2 * tc + 1],
                                           bp[n][0], bp[n][1]);
                            else
                                mma16816(dv[n][tc], va[2 * tc], va[2 * tc + 1], vb[2 * tc], vb[2 * tc + 1],
                                         bp[n][0], bp[n][1]);
                        }
                    }
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) l_run[n] += lsum[n];
                // unit epilogue: acc[c] += (hi + lo) * sigma^V_c * 2^-f, with
                // 2^24 of the subnormal codes and 1 / field scale of the row
                // in the scales
                const float pinv_e = VB ? pinv * kTwo24 : pinv;
#pragma unroll
                for (int tc = 0; tc < 8; ++tc) {
                    const float2 sg = __half22float2(sigv[tc]);
                    const float s0 = sg.x * (pinv_e / (float)VU::vscale(2 * tc));
                    const float s1_ = sg.y * (pinv_e / (float)VU::vscale(2 * tc + 1));
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        acc[n][2 * tc] += (dv[n][tc][0] + dv[n][tc][1]) * s0;
                        acc[n][2 * tc + 1] += (dv[n][tc][2] + dv[n][tc][3]) * s1_;
                    }
                }
                if constexpr (is_nsn(MODE)) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) bsum[n] += __shfl_xor_sync(0xffffffffu, bsum[n], o);
                        if constexpr (MODE == kNsnDq) bsum[n] *= osv;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float2 ov = __half22float2(offv[k]);
                            acco[n][2 * k] += bsum[n] * ov.x;
                            acco[n][2 * k + 1] += bsum[n] * ov.y;
                        }
                    }
                }
                release(uv);
            }
            if (!ok) break;
        }
        if (!ok) break;

        // ---- segment epilogue: the partial of (this warp, pair)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) l_run[n] += __shfl_xor_sync(0xffffffffu, l_run[n], o);
        // code term back to the original domain: acc <- s (.) H acc (the
        // thread's 16 channels 16g + k are the low four index bits, the
        // lanes 4g + t with the same t the high three), plus the offset term
        if constexpr (HAD) {
            const bool sg_ok = a.signs != nullptr;
            const uint4 sraw = sg_ok ? *reinterpret_cast<const uint4*>(a.signs + 16 * g) : make_uint4(0u, 0u, 0u, 0u);
            const int8_t* sgn = reinterpret_cast<const int8_t*>(&sraw);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
#pragma unroll
                for (int m = 1; m < 16; m <<= 1) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        if (k & m) continue;
                        const float x0_ = acc[n][k], x1_ = acc[n][k + m];
                        acc[n][k] = x0_ + x1_;
                        acc[n][k + m] = x0_ - x1_;
                    }
                }
#pragma unroll
                for (int m = 4; m < 32; m <<= 1) {
                    const bool upper = (lane & m) != 0;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float o = __shfl_xor_sync(0xffffffffu, acc[n][k], m);
                        acc[n][k] = upper ? (o - acc[n][k]) : (acc[n][k] + o);
                    }
                }
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (sgn[k] < 0) acc[n][k] = -acc[n][k];
            }
        }
        constexpr int PS = part_stride<D>();
        float* pp = a.part + ((size_t)part_slot(cta, warp, pair) * G) * PS;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int head = 4 * n + t;
            if (head < G) {
                float* pj = pp + (size_t)head * PS;
                if (g == 0) *reinterpret_cast<float4*>(pj) = make_float4(m_ref[n], l_run[n], 0.0f, 0.0f);
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    float4 v4 = make_float4(acc[n][k], acc[n][k + 1], acc[n][k + 2], acc[n][k + 3]);
                    if constexpr (is_nsn(MODE)) {
                        v4.x += acco[n][k]; v4.y += acco[n][k + 1]; v4.z += acco[n][k + 2]; v4.w += acco[n][k + 3];
                    }
                    *reinterpret_cast<float4*>(pj + 4 + 16 * g + k) = v4;
                }
            }
        }
        __syncwarp();
        pos += seg;
    }
    if (!ok) {
        // give the copies still in flight a bounded time to land before the
        // CTA exits; the results of this call are void
        if (lane == 0) report_error(kErrBarrierTimeout);
        for (int u = waited; u < issued; ++u) mbar_wait(&my_bars[u % kRing], (u / kRing) & 1, 1u << 20);
    }
    __syncwarp();
    if (lane < kRing) mbar_inval(&my_bars[lane]);
}

template <int D>
__host__ __device__ constexpr int combine_smem_bytes() {
    return kT * D * 2;  // the residual value rows, fp16
}

// Merge the partials of one (batch, kv head) pair (already in the original
// domain) with its fp16 residual tokens; division by the softmax sum.
// Thread c owns output channel c of every query head.
//
// The kernel is built to keep its chain of dependent memory round trips
// short.  Before waiting for the decode kernel (programmatic dependent
// launch) it loads the queries and all residual keys at once, copies the
// residual value rows to shared memory with cp.async, merges the residual
// tokens as the first softmax chunk and lists the candidate (CTA, warp)
// partial slots.  After the wait, thread i fetches (m, l) of candidate i for
// every head while the accumulators of the first KB candidates are fetched
// in the same round trip.
template <int D, int GP>
__global__ void __launch_bounds__(128) decode_combine_mma_kernel(DecodeArgs a) {
    static_assert(D == 128, "one channel per thread");
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int PS = part_stride<D>();
    constexpr int KB = 64 / GP;  // candidates per batch of accumulator loads (64 floats a thread)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pair = blockIdx.x;
    const int G = a.G;  // <= GP
    const int rlen = a.rlen;
    const int b = pair / a.H, h = pair % a.H;
    extern __shared__ __align__(16) uint8_t comb_raw[];
    __half* s_rv = reinterpret_cast<__half*>(comb_raw);  // [kT][D]
    __shared__ float s_pm[GP][128], s_pl[GP][128];  // candidate m, then weight; l
    __shared__ int s_slot[128];
    __shared__ float s_M[GP], s_L[GP], s_f[GP];
    const float alpha2 = a.scale * kLog2e;
    const int c = tid;

    // ---- everything that does not depend on the decode kernel
    if (rlen > 0) {
        const uint8_t* rv = reinterpret_cast<const uint8_t*>(a.resid[1] + (size_t)pair * kT * D);
        const int nchunk = rlen * (D * 2 / 16);
        for (int i = tid; i < nchunk; i += 128) cp_async16(reinterpret_cast<uint8_t*>(s_rv) + 16 * i, rv + 16 * i);
    }
    if (tid < GP) { s_M[tid] = -INFINITY; s_L[tid] = 0.0f; s_f[tid] = 0.0f; }
    // residual logits on the tensor cores: K rows (fp16) times the queries
    // (fp16, exact); lane (g, t) loads channels 32t .. 32t + 31 of tokens
    // g and g + 8 of each 16-token tile and of query head g; k-step s covers
    // channels 32t + 4s + {0, 1} (k = 2t, 2t + 1) and + {2, 3} (k = 2t + 8, 2t + 9)
    const int g = lane >> 2, t4 = lane & 3;
    uint4 qf[4];
    {
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const __half* qp = a.q + ((size_t)b * a.H * G + (size_t)h * G + g) * D + 32 * t4;
#pragma unroll
        for (int i = 0; i < 4; ++i) qf[i] = (g < G && rlen > 0) ? reinterpret_cast<const uint4*>(qp)[i] : z4;
    }

    // merge one chunk of per-head candidate (m, l) published in s_pm / s_pl:
    // warp w handles heads w, w + 4; weights replace m; s_f gets the rescale
    auto merge_chunk = [&](int n) {
        for (int j = warp; j < G; j += 4) {
            float mx = -INFINITY;
            for (int i = lane; i < n; i += 32) mx = fmaxf(mx, s_pm[j][i]);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float Mo = s_M[j], Mn = fmaxf(Mo, mx);
            float ls = 0.0f;
            for (int i = lane; i < n; i += 32) {
                const float wt = (s_pm[j][i] == -INFINITY) ? 0.0f : exp2f(s_pm[j][i] - Mn);
                s_pm[j][i] = wt;
                ls += wt * s_pl[j][i];
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            if (lane == 0) {
                const float f = (Mo == -INFINITY) ? 0.0f : exp2f(Mo - Mn);
                s_f[j] = f;
                s_L[j] = s_L[j] * f + ls;
                s_M[j] = Mn;
            }
        }
    };

    float A[GP], AO[GP];
#pragma unroll
    for (int j = 0; j < GP; ++j) { A[j] = 0.0f; AO[j] = 0.0f; }
    __syncthreads();

    if (rlen > 0) {
        static_assert(GP <= 8, "one n-tile of query heads");
        const __half* rk = a.resid[0] + (size_t)pair * kT * D;
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(qf);
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        for (int r0 = 16 * warp; r0 < rlen; r0 += 64) {
            const int ta = r0 + g, tb = r0 + g + 8;
            uint4 ka[4], kb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ka[i] = ta < rlen ? reinterpret_cast<const uint4*>(rk + (size_t)ta * D + 32 * t4)[i] : z4;
                kb[i] = tb < rlen ? reinterpret_cast<const uint4*>(rk + (size_t)tb * D + 32 * t4)[i] : z4;
            }
            const uint32_t* wa = reinterpret_cast<const uint32_t*>(ka);
            const uint32_t* wb = reinterpret_cast<const uint32_t*>(kb);
            float d[4];
            mma16816_z(d, wa[0], wb[0], wa[1], wb[1], qw[0], qw[1]);
#pragma unroll
            for (int s2 = 1; s2 < 8; ++s2)
                mma16816(d, wa[2 * s2], wb[2 * s2], wa[2 * s2 + 1], wb[2 * s2 + 1], qw[2 * s2], qw[2 * s2 + 1]);
            // d: (token ta, head 2 t4), (ta, 2 t4 + 1), (tb, 2 t4), (tb, 2 t4 + 1)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int j = 2 * t4 + cc;
                if (j < G) {
                    if (ta < rlen) { s_pm[j][ta] = d[cc] * alpha2; s_pl[j][ta] = 1.0f; }
                    if (tb < rlen) { s_pm[j][tb] = d[2 + cc] * alpha2; s_pl[j][tb] = 1.0f; }
                }
            }
        }
        __syncthreads();
        merge_chunk(rlen);
        cp_async_wait_all();
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < rlen; ++t) {
            const float v = __half2float(s_rv[t * D + c]);
#pragma unroll
            for (int j = 0; j < GP; ++j)
                if (j < G) AO[j] += s_pm[j][t] * v;
        }
    }
    // candidate (CTA, warp) partials of this pair: CTA ranges are contiguous
    const int nctas = (int)(a.nwarps / kNW);
    int c_first = 0, c_last = -1;
    const int px0 = pair * a.nbq, px1 = px0 + a.nbq;  // the pair's blocks [px0, px1)
    const CtaSplit split(a.work > 0 ? a.work : 1, nctas > 0 ? nctas : 1);
    if (a.work > 0 && a.nbq > 0) {
        c_first = split.cta_of(px0);
        c_last = split.cta_of(px1 - 1);
    }
    // warp w of CTA c holds a partial for this pair iff one of its blocks
    // (start(c) + w + kNW i) lies in the pair
    auto has_part = [&](int cta, int w) {
        const int cs = split.start(cta), ce = split.start(cta + 1);
        const int lo = max(cs, px0), hi = min(ce, px1);
        if (hi <= lo) return false;
        const int first = lo + ((w - (lo - cs)) % kNW + kNW) % kNW;  // first block of warp w at or after lo
        return first < hi;
    };
    const float* pbase = a.part + (size_t)part_slot(0, 0, pair) * G * PS;
    const int ncand = (c_last - c_first + 1) * kNW;
    // slot offsets of candidates base .. base + 127 (-1: no partial); they
    // depend on the split only, so the first chunk is listed before the wait
    auto fill_slots = [&](int base) {
        const int i = base + tid;
        const bool valid = i < ncand && has_part(c_first + i / kNW, i % kNW);
        s_slot[tid] = valid ? (int)(part_slot(c_first + i / kNW, i % kNW, pair) - part_slot(0, 0, pair)) : -1;
    };
    fill_slots(0);
    __syncthreads();  // slots listed; the residual phase is done with s_pm

    // ---- the decode kernel's partials
    grid_dep_wait();
    for (int base = 0; base < ncand; base += 128) {
        if (base > 0) {
            fill_slots(base);
            __syncthreads();
        }
        const int n = min(128, ncand - base);
        float av[KB][GP];
        auto load_batch = [&](int i0) {
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                const int o = (i0 + k < n) ? s_slot[i0 + k] : -1;
                const float* pk = pbase + (size_t)(o < 0 ? 0 : o) * G * PS;
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                    const bool use = o >= 0 && j < G;
                    av[k][j] = use ? pk[(size_t)j * PS + 4 + c] : 0.0f;
                }
            }
        };
        // the first accumulators and every candidate's (m, l) in one round trip
        load_batch(0);
        {
            const int off = s_slot[tid];
            float2 ml[GP];
            const float* pk = pbase + (size_t)(off >= 0 ? off : 0) * G * PS;
#pragma unroll
            for (int j = 0; j < GP; ++j)
                ml[j] = (off >= 0 && j < G) ? *reinterpret_cast<const float2*>(pk + (size_t)j * PS)
                                            : make_float2(-INFINITY, 0.0f);
#pragma unroll
            for (int j = 0; j < GP; ++j) {
                if (j < G) { s_pm[j][tid] = ml[j].x; s_pl[j][tid] = ml[j].y; }
            }
        }
        __syncthreads();
        merge_chunk(n);
        __syncthreads();
#pragma unroll
        for (int j = 0; j < GP; ++j) {
            if (j < G) { A[j] *= s_f[j]; AO[j] *= s_f[j]; }
        }
        for (int i0 = 0; i0 < n; i0 += KB) {
            if (i0 > 0) load_batch(i0);
#pragma unroll
            for (int k = 0; k < KB; ++k) {
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                    const float wt = (i0 + k < n && j < G) ? s_pm[j][i0 + k] : 0.0f;
                    A[j] += wt * av[k][j];
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < GP; ++j) {
        if (j >= G) continue;
        const float L = s_L[j];
        a.out[((size_t)b * a.H * G + (size_t)h * G + j) * D + c] = L > 0.0f ? (A[j] + AO[j]) / L : 0.0f;
    }
}

}  // namespace kvq
