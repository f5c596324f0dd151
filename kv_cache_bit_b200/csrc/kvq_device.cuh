// kvq_device.cuh -- device building blocks shared by the libkvq kernels
// (sm_100a): the modes and their stored parameters, PTX wrappers for
// mbarriers and bulk/tensor copies, bounded waits and the error word, and
// the packed-code layout that the quantizer writes and the decode kernels
// read.
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

// kNsnDq: NSN with its side parameters double quantized (the block mean o
// and the token scale s1 kept as 4-bit codes in a per-block record).
enum Mode : int { kNsep = 0, kNaive = 1, kNsn = 2, kNsnDq = 3 };

__host__ __device__ constexpr bool is_nsn(int mode) { return mode == kNsn || mode == kNsnDq; }

// fp16 per-token parameters stored: NSN (s1, s2); NSN with DQ (s2; s1 is in
// the block record); nsep the norm; naive the token scale.
__host__ __device__ constexpr int tok_params(int mode) { return mode == kNsn ? 2 : 1; }

// Block record of the double-quantized NSN side parameters, bytes:
//   [0, D/2)            codes of o: e = q + 8, channel 2j in the low nibble of byte j
//   [D/2, D/2 + 64)     codes of s1: q in 0..15, token 2j in the low nibble of byte j
//   D/2 + 64 + {0,2,4}  fp16 sigma_o, lo, step;  zeros up to a multiple of 16
// o_hat_c = (e_c - 8) sigma_o;  s1_hat_t = lo + q_t step.
template <int D>
__host__ __device__ constexpr int dq_record_bytes() { return (D / 2 + 64 + 6 + 15) / 16 * 16; }
template <int D>
__host__ __device__ constexpr int dq_params_at() { return D / 2 + 64; }
// o_hat of channel c and s1_hat of token t from a block record (as fp32, in
// the oracle's operation order).
template <int D>
__device__ __forceinline__ float dq_o(const uint8_t* rec, int c) {
    const int e = (rec[c >> 1] >> (4 * (c & 1))) & 15;
    return __fmul_rn((float)(e - 8), __half2float(reinterpret_cast<const __half*>(rec + dq_params_at<D>())[0]));
}
template <int D>
__device__ __forceinline__ float dq_s1(const uint8_t* rec, int t) {
    const int q = (rec[D / 2 + (t >> 1)] >> (4 * (t & 1))) & 15;
    const __half* pr = reinterpret_cast<const __half*>(rec + dq_params_at<D>());
    return __fadd_rn(__half2float(pr[1]), __fmul_rn((float)q, __half2float(pr[2])));
}

// fp16 words per block of the NSN offsets array: D means, or the record.
template <int D, int MODE>
__host__ __device__ constexpr int off_words() { return MODE == kNsnDq ? dq_record_bytes<D>() / 2 : D; }

// Sticky device error word, readable with kvq_read_device_errors().
constexpr uint32_t kErrTmaTimeout = 1u;
constexpr uint32_t kErrBarrierTimeout = 2u;
__device__ uint32_t g_error_word = 0;  // the library is a single translation unit

// Poll limit of the bounded waits in the kernels' main loops.  A separate
// test build of the library (KVQ_WAIT_TEST, never the product build) scales
// it by a device variable that a test sets to 0: every such wait then gives
// up at once, so the give-up paths run (error bit, bounded drain of the
// copies in flight) without anything hanging.  The drains keep their limits.
#ifdef KVQ_WAIT_TEST
__device__ uint32_t g_wait_scale = 1;
#define KVQ_WAIT_LIMIT(n) ((n) * g_wait_scale)
#else
#define KVQ_WAIT_LIMIT(n) (n)
#endif

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

// 2-D tiled TMA store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the committed bulk stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// 1-D bulk copy global -> shared (no multicast); size and both addresses
// must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void report_error(uint32_t bit) { atomicOr(&g_error_word, bit); }

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start before the kernel ahead of it in the stream has
// finished; grid_dep_wait() returns once that kernel has completed and its
// memory is visible (at once when the launch attribute is absent), and
// grid_dep_launch() lets the kernel behind this one be scheduled early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- packing

template <int D, int BITS>
struct RowLayout {
    static constexpr int kBytes = D * BITS / 8;  // 2/3/4 bits per code
    static constexpr int kWords = kBytes / 4;
    static constexpr int kOff = 1 << (BITS - 1);  // offset-binary bias
    static constexpr int kQmax = (1 << (BITS - 1)) - 1;
};

// A packed token row holds the offset-binary codes e[c] (1 .. 2^BITS - 1)
// in 32-bit words, little-endian byte order:
//   INT4 byte j = e[2j] | e[2j+1] << 4
//   INT2 byte j = e[4j] | e[4j+1] << 2 | e[4j+2] << 4 | e[4j+3] << 6
//   INT3 plane of (e & 3) in the INT2 layout (D/4 bytes), then a plane whose
//        bit i of byte j is bit 2 of e[8j+i] (D/8 bytes)
// (V rows of head dim 128 are further pair-interleaved, see pairv_layout).

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

// ---------------------------------------------------------------- value rows
// V code rows of head dim 128 are stored pair-interleaved, the layout the
// decode kernel's value operand wants (two tokens' codes of one channel in
// one 32-bit register): the rows of tokens 2k and 2k + 1 of a block form a
// pair block of 2 * row_bytes bytes whose 32-bit word u holds the 2-byte unit
// u (bytes 2u, 2u + 1) of row 2k in its low half and of row 2k + 1 in its
// high half.  For INT4 the 16-byte chunk c of pair block k sits at chunk
// c ^ (2 (k & 1)), which spreads a quarter warp's 16-byte loads over the
// banks; token 2k + s fills the s-th row_bytes half of its pair block.
template <int D>
__host__ __device__ constexpr bool pairv_layout() { return D == 128; }
template <int BITS>
__host__ __device__ constexpr int pairv_chunk_xor(int k) { return BITS == 4 ? 2 * (k & 1) : 0; }

}  // namespace kvq
