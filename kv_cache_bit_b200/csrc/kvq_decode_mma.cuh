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

constexpr int kUT = 64;  // tokens per staging unit (half a block)

// A unit is one tensor's half block: packed codes and per-token parameters of
// 64 tokens; the first half also carries the block's channel scales and NSN
// channel means.
template <int D, int BITS, int MODE>
struct SlotLayout {
    static constexpr int kRB = D * BITS / 8;
    static constexpr int kNtok = (MODE == kNsn) ? 2 : 1;
    static constexpr int kCodes = 0;
    static constexpr int kTok = kUT * kRB;
    static constexpr int kChan = kTok + kUT * kNtok * 2;
    static constexpr int kOff = kChan + ((MODE != kNaive) ? D * 2 : 0);
    static constexpr int kBytesLo = kOff + ((MODE == kNsn) ? D * 2 : 0);  // first half
    static constexpr int kBytesHi = kChan;                                 // second half
    static constexpr int kStride = (kBytesLo + 127) / 128 * 128;
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

// Token held by fragment row r (0..15) of a 16-token tile: rows 2k and 2k + 1
// swap when k is odd.  Thread quads then read token rows of alternating
// parity, which spreads the V-side loads over both halves of the banks.
__device__ __forceinline__ int tile_tok(int r) { return r ^ ((r >> 1) & 1); }

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
template <int D, int BITS, int MODE, bool HAD, int GP>
__global__ void __launch_bounds__(kNW * 32) decode_mma_kernel(DecodeArgs a) {
    static_assert(D == 128, "tensor-core decode is built for head dim 128");
    using SL = SlotLayout<D, BITS, MODE>;
    constexpr int NT = GP / 4;  // n-tiles (heads per thread)
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
    __shared__ float s_q[GP][D];  // queries (original domain)
    // rotated queries times the head's power-of-two scale; element c of head j
    // at j * kQS + c + c / 32, so the four 32-channel slices of four heads fall
    // in distinct banks
    constexpr int kQS = D + 4;
    __shared__ float s_qs[GP * kQS];
    __shared__ float s_qscale[GP];

    if (tid < kNW * kRing) mbar_init(&bars[tid], 1);
    fence_mbar_init();
    // ---- prologue: each warp rotates heads warp, warp + kNW, ... (lane owns 4 channels)
    for (int j = warp; j < GP; j += kNW) {
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c = 4 * lane + k;
            const float qv = (j < G) ? __half2float(a.q[((size_t)b * a.H * G + (size_t)h * G + j) * D + c]) : 0.0f;
            s_q[j][c] = qv;
            v[k] = (HAD && a.signs != nullptr && a.signs[c] < 0) ? -qv : qv;
        }
        if constexpr (HAD) {
            float x0 = v[0] + v[1], x1 = v[0] - v[1], x2 = v[2] + v[3], x3 = v[2] - v[3];
            v[0] = x0 + x2; v[2] = x0 - x2; v[1] = x1 + x3; v[3] = x1 - x3;
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
            const int c = 4 * lane + k;
            s_qs[j * kQS + c + (c >> 5)] = v[k] * qsc;
        }
        if (lane == 0) s_qscale[j] = qsc;
    }
    __syncthreads();

    // ---- this warp's blocks: units 4i + k = (K lo, V lo, K hi, V hi) of block i
    const int blk_begin = split * a.bps;
    const int blk_end = min(a.nbq, blk_begin + a.bps);
    const int nmine = blk_end > blk_begin + warp ? (blk_end - blk_begin - warp + kNW - 1) / kNW : 0;
    const int nunits = 4 * nmine;
    uint8_t* my_ring = ring + warp * kRing * SL::kStride;
    uint64_t* my_bars = bars + warp * kRing;

    auto issue = [&](int u) {
        const int blk = blk_begin + warp + kNW * (u >> 2);
        const int ten = u & 1;
        const int half = (u >> 1) & 1;
        uint8_t* slot = my_ring + (u % kRing) * SL::kStride;
        uint64_t* bar = &my_bars[u % kRing];
        const size_t row0 = (size_t)bh * a.cap + (size_t)blk * kT + (size_t)half * kUT;
        const size_t bi = ((size_t)bh * nb_cap + blk) * D;
        mbar_expect_tx(bar, half ? SL::kBytesHi : SL::kBytesLo);
        bulk_load(slot + SL::kCodes, (ten ? a.codes[1] : a.codes[0]) + row0 * SL::kRB, kUT * SL::kRB, bar);
        bulk_load(slot + SL::kTok, (ten ? a.tok[1] : a.tok[0]) + row0 * SL::kNtok, kUT * SL::kNtok * 2, bar);
        if (!half) {
            if (PCH) bulk_load(slot + SL::kChan, (ten ? a.chan[1] : a.chan[0]) + bi, D * 2, bar);
            if (MODE == kNsn) bulk_load(slot + SL::kOff, (ten ? a.off[1] : a.off[0]) + bi, D * 2, bar);
        }
    };
    int issued = min(kRing, nunits);
    if (lane == 0) {
        for (int u = 0; u < issued; ++u) issue(u);
    }
    int waited = 0;
    bool ok = true;
    auto wait_unit = [&](int u) -> bool {
        if (!mbar_wait(&my_bars[u % kRing], (u / kRing) & 1, 1u << 26)) return false;
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
            issued = u + kRing + 1;
        }
    };

    // ---- persistent per-thread state: heads 4n + t, channels [16g, 16g + 16)
    // Softmax weights are taken against a reference max m_ref that only moves
    // when a tile's logit exceeds it by more than kTau (log2 units), so that
    // p <= 2^kTau and most tiles need no rescale.
    constexpr float kTau = 8.0f;
    float m_ref[NT], l_run[NT];
    float acc[NT][16], acco[NT][16];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        m_ref[n] = -INFINITY;
        l_run[n] = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) { acc[n][k] = 0.0f; acco[n][k] = 0.0f; }
    }
    float kcol[NT];  // 1 / (the head's power-of-two scale)
#pragma unroll
    for (int n = 0; n < NT; ++n) kcol[n] = 1.0f / s_qscale[4 * n + t];
    // the B column this thread feeds in each n-tile: head 4n + g/2, part g%2
    const bool blo = (g & 1) != 0;
    const float alpha2 = a.scale * kLog2e;
    // token of fragment rows g and g + 8 inside a 16-token tile
    const int tr0 = tile_tok(g), tr1 = 8 + tile_tok(g);
    // V fragment rows 2t, 2t+1, 2t+8, 2t+9
    const int vr0 = tile_tok(2 * t), vr1 = tile_tok(2 * t + 1);

    uint32_t bq[NT][16];
    float qoK[NT];
    __half2 sigv[8], offv[8];
    for (int it = 0; it < nmine; ++it) {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int uk = 4 * it + 2 * half, uv = uk + 1;
            if (!wait_unit(uk)) { ok = false; break; }
            uint8_t* sk = my_ring + (uk % kRing) * SL::kStride;
            if (half == 0) {
                // B fragments: q' = qs * sigma^K as (hi, lo) fp16 parts
                const __half* sig = reinterpret_cast<const __half*>(sk + SL::kChan) + 32 * t;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const float* qrow = &s_qs[(4 * n + (g >> 1)) * kQS + 33 * t];
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const int ca = KUnpack<BITS>::ca(p), cb = KUnpack<BITS>::cb(p);
                        const float fa = qrow[ca] * (PCH ? __half2float(sig[ca]) : 1.0f);
                        const float fb = qrow[cb] * (PCH ? __half2float(sig[cb]) : 1.0f);
                        const __half2 hh = __floats2half2_rn(fa, fb);
                        if (blo) {
                            const float2 hf = __half22float2(hh);
                            bq[n][p] = cvt_h2(fa - hf.x, fb - hf.y);
                        } else {
                            bq[n][p] = *reinterpret_cast<const uint32_t*>(&hh);
                        }
                    }
                }
                if constexpr (MODE == kNsn) {
                    const __half* okp = reinterpret_cast<const __half*>(sk + SL::kOff) + 16 * g;
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float s = 0.0f;
#pragma unroll
                        for (int k = 0; k < 16; ++k) s += s_q[4 * n + t][16 * g + k] * __half2float(okp[k]);
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                        qoK[n] = s;
                    }
                }
            }
            if (!wait_unit(uv)) { ok = false; break; }
            uint8_t* sv = my_ring + (uv % kRing) * SL::kStride;
            if (half == 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    sigv[k] = PCH ? reinterpret_cast<const __half2*>(sv + SL::kChan)[8 * g + k]
                                  : __floats2half2_rn(1.f, 1.f);
                    offv[k] = (MODE == kNsn) ? reinterpret_cast<const __half2*>(sv + SL::kOff)[8 * g + k]
                                             : __floats2half2_rn(0.f, 0.f);
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
                } else {
                    v = __half2float(tv[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                }
                numax = fmaxf(numax, v);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) numax = fmaxf(numax, __shfl_xor_sync(0xffffffffu, numax, o));
            const int fexp = numax > 0.0f ? 13 - (int)kTau - ceil_log2(numax) : 0;
            const float pscale = pow2i(fexp), pinv = pow2i(-fexp);
            float dv[NT][8][4];
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k) dv[n][i][k] = 0.0f;
            float lsum[NT], bsum[NT];
#pragma unroll
            for (int n = 0; n < NT; ++n) { lsum[n] = 0.0f; bsum[n] = 0.0f; }
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                // ---- scores of the tile's 16 tokens
                uint32_t pa[16], pb[16];
                KUnpack<BITS>::run(sk + SL::kCodes + (16 * m4 + tr0) * SL::kRB, t, pa);
                KUnpack<BITS>::run(sk + SL::kCodes + (16 * m4 + tr1) * SL::kRB, t, pb);
                float l2[NT][2];
                bool over = false;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int s = 0; s < 8; s += 2) {
                        mma16816(d0, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], bq[n][2 * s],
                                 bq[n][2 * s + 1]);
                        mma16816(d1, pa[2 * s + 2], pb[2 * s + 2], pa[2 * s + 3], pb[2 * s + 3], bq[n][2 * s + 2],
                                 bq[n][2 * s + 3]);
                    }
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int tok = 16 * m4 + (r ? tr1 : tr0);
                        const float sv_ = (d0[2 * r] + d0[2 * r + 1]) + (d1[2 * r] + d1[2 * r + 1]);
                        float kap, add = 0.0f;
                        if constexpr (MODE == kNsn) {
                            const float2 s12 = __half22float2(reinterpret_cast<const __half2*>(tk)[tok]);
                            kap = s12.x * s12.y * (HAD ? 1.0f : a.sqd);
                            add = s12.x * qoK[n];
                        } else {
                            kap = __half2float(tk[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                        }
                        l2[n][r] = (sv_ * (kap * kcol[n]) + add) * alpha2;
                        over |= l2[n][r] > m_ref[n] + kTau;
                    }
                }
                // ---- rare: move the reference max up and rescale what was accumulated
                if (__any_sync(0xffffffffu, over)) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float mx = fmaxf(l2[n][0], l2[n][1]);
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        const float mn = fmaxf(m_ref[n], mx);
                        const float corr = fast_exp2(m_ref[n] - mn);
                        m_ref[n] = mn;
                        l_run[n] *= corr;
                        lsum[n] *= corr;
                        bsum[n] *= corr;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            acc[n][k] *= corr;
                            if (MODE == kNsn) acco[n][k] *= corr;
                        }
#pragma unroll
                        for (int i = 0; i < 8; ++i)
#pragma unroll
                            for (int k = 0; k < 4; ++k) dv[n][i][k] *= corr;
                    }
                }
                // ---- P' = p * nu (scaled), as (hi, lo) rows, moved into the B layout
                uint32_t bp[NT][2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int tok = 16 * m4 + (r ? tr1 : tr0);
                    float nu, s1o = 0.0f;
                    if constexpr (MODE == kNsn) {
                        const float2 s12 = __half22float2(reinterpret_cast<const __half2*>(tv)[tok]);
                        s1o = s12.x;
                        nu = s12.x * s12.y * (HAD ? 1.0f : a.sqd);
                    } else {
                        nu = __half2float(tv[tok]) * ((MODE == kNsep && HAD) ? a.rsqd : 1.0f);
                    }
                    nu *= pscale;
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const float p = fast_exp2(l2[n][r] - m_ref[n]);
                        lsum[n] += p;
                        if constexpr (MODE == kNsn) bsum[n] += p * s1o;
                        bp[n][r] = movmatrix_t(split_h2(p * nu));
                    }
                }
                // ---- values
                uint32_t va[16], vb[16];
                const uint8_t* vbase = sv + SL::kCodes + (16 * m4) * SL::kRB;
                VUnpack<BITS>::run(vbase + vr0 * SL::kRB, vbase + vr1 * SL::kRB, g, va);
                VUnpack<BITS>::run(vbase + (8 + vr0) * SL::kRB, vbase + (8 + vr1) * SL::kRB, g, vb);
#pragma unroll
                for (int tc = 0; tc < 8; ++tc) {
#pragma unroll
                    for (int n = 0; n < NT; ++n)
                        mma16816(dv[n][tc], va[2 * tc], va[2 * tc + 1], vb[2 * tc], vb[2 * tc + 1], bp[n][0], bp[n][1]);
                }
            }
            release(uk);
#pragma unroll
            for (int n = 0; n < NT; ++n) l_run[n] += lsum[n];
            // unit epilogue: acc[c] += (hi + lo) * sigma^V_c * 2^-f
#pragma unroll
            for (int tc = 0; tc < 8; ++tc) {
                const float2 sg = __half22float2(sigv[tc]);
                const float s0 = sg.x * pinv, s1_ = sg.y * pinv;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    acc[n][2 * tc] += (dv[n][tc][0] + dv[n][tc][1]) * s0;
                    acc[n][2 * tc + 1] += (dv[n][tc][2] + dv[n][tc][3]) * s1_;
                }
            }
            if constexpr (MODE == kNsn) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) bsum[n] += __shfl_xor_sync(0xffffffffu, bsum[n], o);
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
    float m_run[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) m_run[n] = m_ref[n];
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
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) l_run[n] += __shfl_xor_sync(0xffffffffu, l_run[n], o);
    __syncthreads();  // every warp is done with its ring; reuse it for the merge
    float* mw = reinterpret_cast<float*>(smem_raw);   // [kNW][kGMax] running max
    float* lw = mw + kNW * kGMax;                     // [kNW][kGMax] sums
    float* aw = lw + kNW * kGMax;                     // [kNW][kGMax][D] code-term accumulators
    float* ow = aw + kNW * kGMax * D;                 // [kNW][kGMax][D] original-domain accumulators
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = 4 * n + t;
        if (g == 0) {
            mw[warp * kGMax + head] = m_run[n];
            lw[warp * kGMax + head] = l_run[n];
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            aw[(warp * kGMax + head) * D + 16 * g + k] = acc[n][k];
            ow[(warp * kGMax + head) * D + 16 * g + k] = (MODE == kNsn) ? acco[n][k] : 0.0f;
        }
    }
    __syncthreads();

    // residual tokens (fp16), handled by the last split on CUDA cores
    float* pp = a.part + ((size_t)bh * a.nsplit + split) * G * (2 + 2 * D);
    const bool do_res = (split == a.nsplit - 1) && a.rlen > 0;
    float* rl = ow + kNW * kGMax * D;  // [kGMax][kT] residual logits / weights
    float* rm = rl + kGMax * kT;       // [kGMax] residual max, [kGMax] sum
    if (do_res) {
        const __half* rk = a.resid[0] + (size_t)bh * kT * D;
        // warp w scores tokens w, w + kNW, ...; lanes split the channels
        for (int tr = warp; tr < kT; tr += kNW) {
            float x[4];
            if (tr < a.rlen) {
                const float2 x01 = __half22float2(reinterpret_cast<const __half2*>(rk + (size_t)tr * D)[2 * lane]);
                const float2 x23 = __half22float2(reinterpret_cast<const __half2*>(rk + (size_t)tr * D)[2 * lane + 1]);
                x[0] = x01.x; x[1] = x01.y; x[2] = x23.x; x[3] = x23.y;
            }
            for (int j = 0; j < G; ++j) {
                float s = -INFINITY;
                if (tr < a.rlen) {
                    s = 0.0f;
#pragma unroll
                    for (int k = 0; k < 4; ++k) s += s_q[j][4 * lane + k] * x[k];
#pragma unroll
                    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                    s *= alpha2;
                }
                if (lane == 0) rl[j * kT + tr] = s;
            }
        }
        __syncthreads();
        for (int j = warp; j < G; j += kNW) {
            float mx = -INFINITY;
            for (int i = lane; i < kT; i += 32) mx = fmaxf(mx, rl[j * kT + i]);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float sm = 0.0f;
            for (int i = lane; i < kT; i += 32) {
                const float p = (rl[j * kT + i] == -INFINITY) ? 0.0f : fast_exp2(rl[j * kT + i] - mx);
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
