// kvq_device.cuh -- device building blocks shared by the libkvq kernels
// (sm_100a): PTX wrappers for mbarriers and bulk/tensor copies, the
// per-token quantizer that one CTA of 128 threads runs over a 128-token
// block (one thread per token row), and the packed-code layout.
//
// Arithmetic that decides a stored bit (norms, means, scales, codes) uses the
// explicitly rounded intrinsics (__fmul_rn, __fadd_rn, __fdiv_rn, __fsqrt_rn,
// __fmaf_rn) so that the compiler never contracts or reorders it.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace kvq {

constexpr int kT = 128;  // tokens per scale block

enum Mode : int { kNsep = 0, kNaive = 1, kNsn = 2 };

// Sticky device error word, readable with kvq_read_device_errors().
constexpr uint32_t kErrTmaTimeout = 1u;
constexpr uint32_t kErrBarrierTimeout = 2u;
__device__ uint32_t g_error_word = 0;  // the library is a single translation unit

// ---------------------------------------------------------------- PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One bounded wait on phase `parity`.  Returns false if the phase did not
// complete within `max_iter` polls (each poll may suspend the thread for a
// short, hardware-chosen time).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t max_iter) {
    uint32_t addr = smem_u32(bar);
    for (uint32_t it = 0; it < max_iter; ++it) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n"
            " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// 2-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy global -> shared (no multicast); size and both addresses
// must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void report_error(uint32_t bit) { atomicOr(&g_error_word, bit); }

// ---------------------------------------------------------------- packing

template <int D, int BITS>
struct RowLayout {
    static constexpr int kBytes = D * BITS / 8;  // 2/3/4 bits per code
    static constexpr int kWords = kBytes / 4;
    static constexpr int kOff = 1 << (BITS - 1);  // offset-binary bias
    static constexpr int kQmax = (1 << (BITS - 1)) - 1;
};

// Pack offset-binary codes e[c] (1 .. 2^BITS - 1) of one token row into
// 32-bit words, little-endian byte order:
//   INT4 byte j = e[2j] | e[2j+1] << 4
//   INT2 byte j = e[4j] | e[4j+1] << 2 | e[4j+2] << 4 | e[4j+3] << 6
//   INT3 plane of (e & 3) in the INT2 layout (D/4 bytes), then a plane whose
//        bit i of byte j is bit 2 of e[8j+i] (D/8 bytes)
template <int D, int BITS>
__device__ __forceinline__ void pack_row(const uint32_t (&e)[D], uint32_t (&w)[RowLayout<D, BITS>::kWords]) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int k = 0; k < D / 8; ++k) {
            uint32_t v = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) v |= (e[8 * k + i] & 15u) << (4 * i);
            w[k] = v;
        }
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            uint32_t v = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) v |= (e[16 * k + i] & 3u) << (2 * i);
            w[k] = v;
        }
    } else {
        static_assert(BITS == 3, "bits");
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            uint32_t v = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) v |= (e[16 * k + i] & 3u) << (2 * i);
            w[k] = v;
        }
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
            uint32_t v = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) v |= ((e[32 * k + i] >> 2) & 1u) << i;
            w[D / 16 + k] = v;
        }
    }
}

// Offset-binary code of channel c from a packed row held as 32-bit words.
template <int D, int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t* w, int c) {
    if constexpr (BITS == 4) return (w[c >> 3] >> (4 * (c & 7))) & 15u;
    else if constexpr (BITS == 2) return (w[c >> 4] >> (2 * (c & 15))) & 3u;
    else return ((w[c >> 4] >> (2 * (c & 15))) & 3u) | (((w[D / 16 + (c >> 5)] >> (c & 31)) & 1u) << 2);
}

// Store / load a packed row with the widest aligned vector access.
template <int NW>
__device__ __forceinline__ void store_words(uint8_t* dst, const uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NW / 4; ++k)
            reinterpret_cast<uint4*>(dst)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    } else if constexpr (NW % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NW / 2; ++k) reinterpret_cast<uint2*>(dst)[k] = make_uint2(w[2 * k], w[2 * k + 1]);
    } else {
#pragma unroll
        for (int k = 0; k < NW; ++k) reinterpret_cast<uint32_t*>(dst)[k] = w[k];
    }
}

template <int NW>
__device__ __forceinline__ void load_words(const uint8_t* src, uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NW / 4; ++k) {
            uint4 v = reinterpret_cast<const uint4*>(src)[k];
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
    } else if constexpr (NW % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NW / 2; ++k) {
            uint2 v = reinterpret_cast<const uint2*>(src)[k];
            w[2 * k] = v.x; w[2 * k + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int k = 0; k < NW; ++k) w[k] = reinterpret_cast<const uint32_t*>(src)[k];
    }
}

// ---------------------------------------------------------------- arithmetic

// fp32 pairwise sum of squares over v[OFF .. OFF+N): sum(first half) +
// sum(second half), recursively; squares and sums separately rounded.
template <int OFF, int N, int D>
__device__ __forceinline__ float pw_sumsq(const float (&v)[D]) {
    if constexpr (N == 1) return __fmul_rn(v[OFF], v[OFF]);
    else return __fadd_rn(pw_sumsq<OFF, N / 2>(v), pw_sumsq<OFF + N / 2, N / 2>(v));
}

// In-register unnormalized Walsh-Hadamard butterflies, strides H = 1, 2, ...,
// D/2 in that order (compile-time recursion keeps every index static).
template <int H, int D>
__device__ __forceinline__ void fwht_stage(float (&v)[D]) {
#pragma unroll
    for (int i = 0; i < D; i += 2 * H) {
#pragma unroll
        for (int j = 0; j < H; ++j) {
            const float a = v[i + j], b = v[i + j + H];
            v[i + j] = __fadd_rn(a, b);
            v[i + j + H] = __fsub_rn(a, b);
        }
    }
    if constexpr (2 * H < D) fwht_stage<2 * H, D>(v);
}

template <int D>
__device__ __forceinline__ void fwht_reg(float (&v)[D]) {
    fwht_stage<1, D>(v);
}

// Round-half-even of the exact product u * inv, clamped to [-qmax, qmax],
// returned as the offset-binary code.  The fused multiply-add rounds the
// exact product plus 1.5 * 2^23 once to an integer (ties to even); the
// subtraction is exact while |u * inv| < 2^22, and larger magnitudes clamp.
template <int QMAX>
__device__ __forceinline__ uint32_t code_of(float u, float inv) {
    const float kMagic = 12582912.0f;  // 1.5 * 2^23
    float r = __fsub_rn(__fmaf_rn(u, inv, kMagic), kMagic);
    r = fminf(fmaxf(r, -(float)QMAX), (float)QMAX);
    return static_cast<uint32_t>(static_cast<int>(r) + QMAX + 1);
}

// ---------------------------------------------------------------- the quantizer

// Shared-memory scratch of one quantizer CTA.
template <int D>
struct QuantSmem {
    // fp32 [128][D] transpose buffer (NSN column means), swizzled by 16-byte
    // chunk: chunk k of row t lives at chunk k ^ (t & (D/4 - 1)).
    static constexpr int kRedFloats = kT * D;
    float* red;
    float* vec;        // [D] broadcast vector (means, reciprocal scales)
    uint32_t* wmax;    // [4][D] per-warp channel maxima (float bits)
    uint32_t* sgn;     // [D] sign masks (0 or 0x80000000) of the rotation
};

// Output pointers of one (tensor, batch, head, block).
struct QuantOut {
    uint8_t* codes;  // [128][row_bytes] rows of this block
    __half* tok;     // [128][ntok]
    __half* chan;    // [D] (PER_CHANNEL)
    __half* off;     // [D] (NSN)
};

// Quantize the 128 token rows of one block; thread t (0..127) holds row t in
// v[] (fp32 widened from fp16) and all 128 threads of the CTA must call this.
//   nsep:  n = ||x||, u = H(s (.) x) * (c0 / n)
//   NSN:   s1 = ||x|| rsqd, a = x (sqd / ||x||), o = block mean of a (fp16),
//          b = a - o, s2 = ||b|| rsqd, u = H(s (.) b) * (c0 / ||b||)
//   naive: u = x
// with c0 = rsqd under HADAMARD, else 1; then sigma = fp16(max|u| / qmax)
// per channel over the block (per token for naive) and codes
// rne(u * (1/sigma)) clamped.
template <int D, int BITS, int MODE, bool HAD>
__device__ __forceinline__ void quantize_rows(float (&v)[D], const int t, const QuantSmem<D>& sm, const QuantOut& out,
                                              const float rsqd, const float sqd) {
    using L = RowLayout<D, BITS>;
    const float c0 = HAD ? rsqd : 1.0f;
    float kscale = 1.0f;

    if constexpr (MODE == kNsn) {
        const float n1 = __fsqrt_rn(pw_sumsq<0, D>(v));
        const float s1 = __fmul_rn(n1, rsqd);
        const float r1 = n1 > 0.0f ? __fdiv_rn(sqd, n1) : 0.0f;
#pragma unroll
        for (int c = 0; c < D; ++c) v[c] = __fmul_rn(v[c], r1);
        // transpose through shared memory for the per-channel block means
        constexpr int NCH = D / 4;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            const int pk = k ^ (t & (NCH - 1));
            reinterpret_cast<float4*>(sm.red + t * D)[pk] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        }
        __syncthreads();
        {
            // thread -> (column c, token half). For D = 128 every thread sums
            // one full column; for D = 64 two threads split the column and
            // their halves are added last (the top split of the pairwise tree).
            constexpr int PER = (D == 128) ? 128 : 64;
            const int c = t % D;
            const int tbase = (t / D) * PER;
            float acc[8];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int tt = tbase + i;
                const int pk = (c >> 2) ^ (tt & (NCH - 1));
                float cur = sm.red[tt * D + pk * 4 + (c & 3)];
#pragma unroll
                for (int l = 0; l < 7; ++l) {
                    if ((i >> l) & 1) cur = __fadd_rn(acc[l], cur);
                    else { acc[l] = cur; break; }
                }
                if (i == PER - 1) acc[7] = cur;
            }
            if constexpr (D == 128) {
                const float o = __fmul_rn(acc[7], 1.0f / 128.0f);
                const __half o16 = __float2half_rn(o);
                out.off[c] = o16;
                sm.vec[c] = __half2float(o16);
            } else {
                // halves meet in smem: lower half writes, upper half adds
                __syncthreads();
                if (t >= D) sm.vec[c] = acc[7];
                __syncthreads();
                if (t < D) {
                    const float o = __fmul_rn(__fadd_rn(acc[7], sm.vec[c]), 1.0f / 128.0f);
                    const __half o16 = __float2half_rn(o);
                    out.off[c] = o16;
                    sm.vec[c] = __half2float(o16);
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < D; ++c) v[c] = __fsub_rn(v[c], sm.vec[c]);
        const float n2 = __fsqrt_rn(pw_sumsq<0, D>(v));
        const float s2 = __fmul_rn(n2, rsqd);
        kscale = n2 > 0.0f ? __fdiv_rn(c0, n2) : 0.0f;
        __half2 sp = __halves2half2(__float2half_rn(s1), __float2half_rn(s2));
        reinterpret_cast<__half2*>(out.tok)[t] = sp;
    } else if constexpr (MODE == kNsep) {
        const float n = __fsqrt_rn(pw_sumsq<0, D>(v));
        out.tok[t] = __float2half_rn(n);
        kscale = n > 0.0f ? __fdiv_rn(c0, n) : 0.0f;
    } else {
        kscale = c0;
    }

    if constexpr (HAD) {
#pragma unroll
        for (int c = 0; c < D; ++c) v[c] = __uint_as_float(__float_as_uint(v[c]) ^ sm.sgn[c]);
        fwht_reg<D>(v);
    }
    if constexpr (MODE != kNaive || HAD) {
#pragma unroll
        for (int c = 0; c < D; ++c) v[c] = __fmul_rn(v[c], kscale);
    }

    uint32_t e[D];
    if constexpr (MODE == kNaive) {
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < D; ++c) m = fmaxf(m, fabsf(v[c]));
        const __half s16 = __float2half_rn(__fdiv_rn(m, (float)L::kQmax));
        out.tok[t] = s16;
        const float sf = __half2float(s16);
        const float inv = sf > 0.0f ? __fdiv_rn(1.0f, sf) : 0.0f;
#pragma unroll
        for (int c = 0; c < D; ++c) e[c] = code_of<L::kQmax>(v[c], inv);
    } else {
        // per-channel absmax over the block: warp max, then across warps
        const int warp = t >> 5, lane = t & 31;
#pragma unroll
        for (int c = 0; c < D; ++c) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v[c])));
            if (lane == (c & 31)) sm.wmax[warp * D + c] = m;
        }
        __syncthreads();
        if (t < D) {
            const float m = fmaxf(fmaxf(__uint_as_float(sm.wmax[t]), __uint_as_float(sm.wmax[D + t])),
                                  fmaxf(__uint_as_float(sm.wmax[2 * D + t]), __uint_as_float(sm.wmax[3 * D + t])));
            const __half s16 = __float2half_rn(__fdiv_rn(m, (float)L::kQmax));
            out.chan[t] = s16;
            const float sf = __half2float(s16);
            sm.vec[t] = sf > 0.0f ? __fdiv_rn(1.0f, sf) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < D; ++c) e[c] = code_of<L::kQmax>(v[c], sm.vec[c]);
    }
    uint32_t w[L::kWords];
    pack_row<D, BITS>(e, w);
    store_words<L::kWords>(out.codes + (size_t)t * L::kBytes, w);
}

}  // namespace kvq
