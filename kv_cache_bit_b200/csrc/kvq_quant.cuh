// kvq_quant.cuh -- block quantizer, residual append/flush and dequantizer
// kernels (sm_100a).  Included once, by kvq_api.cu.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct QuantArgs {
    // per tensor (0 = K, 1 = V); layouts as in kvq.h
    uint8_t* codes[2];
    __half* tok[2];
    __half* chan[2];
    __half* off[2];
    const int8_t* signs;
    int H;           // kv heads
    int bh;          // batch * kv heads
    int cap;         // cache capacity (tokens)
    int ntok;        // tokens in this call (multiple of 128)
    int blk0;        // first destination block
    float rsqd, sqd; // (float)(1/sqrt(d)), (float)sqrt(d)
};

// Shared memory of a quantizer CTA: three regions of one fp16 tile each
// (128 x D x 2 bytes, which is also half of the fp32 transpose buffer), the
// small vectors and three mbarriers.
template <int D>
__host__ __device__ constexpr int quant_region_bytes() {
    return kT * D * 2;
}

template <int D>
__host__ __device__ constexpr int quant_smem_bytes() {
    // 1024 B alignment slack + 3 regions + vec + group partials + token vector + sign masks + mbarriers
    return 1024 + 3 * quant_region_bytes<D>() + D * 4 + kGpartBytes + kT * 4 + D * 4 + 3 * 8;
}

template <int D>
__device__ __forceinline__ QuantSmem<D> carve_quant_smem(uint8_t* base, uint64_t*& bar, uint8_t*& regions) {
    uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(base) + 1023) & ~uintptr_t(1023));
    QuantSmem<D> sm;
    regions = p;
    sm.tile = p;
    sm.red_lo = reinterpret_cast<float*>(p + quant_region_bytes<D>());
    sm.red_hi = reinterpret_cast<float*>(p + 2 * quant_region_bytes<D>());
    p += 3 * quant_region_bytes<D>();
    sm.vec = reinterpret_cast<float*>(p);
    p += D * 4;
    sm.gpart = reinterpret_cast<float*>(p);
    p += kGpartBytes;
    sm.tokv = reinterpret_cast<float*>(p);
    p += kT * 4;
    sm.sgn2 = reinterpret_cast<uint32_t*>(p);
    p += D * 4;
    bar = reinterpret_cast<uint64_t*>(p);
    return sm;
}

template <int D, int BITS, int MODE, bool HAD>
__device__ __forceinline__ QuantOut quant_out(const QuantArgs& a, int tensor, int bh, int blk) {
    using L = RowLayout<D, BITS>;
    const int ntk = (MODE == kNsn) ? 2 : 1;
    const int nb = a.cap / kT;
    QuantOut o;
    // select with ternaries: a runtime index into the parameter arrays would
    // copy them to local memory
    const bool v = tensor != 0;
    o.codes = (v ? a.codes[1] : a.codes[0]) + ((size_t)bh * a.cap + (size_t)blk * kT) * L::kBytes;
    o.tok = (v ? a.tok[1] : a.tok[0]) + ((size_t)bh * a.cap + (size_t)blk * kT) * ntk;
    o.chan = (MODE != kNaive) ? (v ? a.chan[1] : a.chan[0]) + ((size_t)bh * nb + blk) * D : nullptr;
    o.off = (MODE == kNsn) ? (v ? a.off[1] : a.off[0]) + ((size_t)bh * nb + blk) * D : nullptr;
    o.stage = nullptr;
    o.pairv = pairv_layout<D>() && v;
    return o;
}

template <int D, bool HAD>
__device__ __forceinline__ void load_signs(const QuantArgs& a, const QuantSmem<D>& sm, int t) {
    if constexpr (HAD) {
        if (t < D / 2) {
            const bool n0 = a.signs != nullptr && a.signs[2 * t] < 0;
            const bool n1 = a.signs != nullptr && a.signs[2 * t + 1] < 0;
            sm.sgn2[t] = (n0 ? 0x8000u : 0u) | (n1 ? 0x80000000u : 0u);
        }
    }
}

// Widen 8 fp16 channels of the low half (lo) and the matching 8 of the high
// half (hi) into pairs P[8q .. 8q+8), after the rotation's sign flips.
template <int D, bool HAD>
__device__ __forceinline__ void widen_chunk(uint4 lo, uint4 hi, int q, const QuantSmem<D>& sm, f2_t (&P)[D / 2]) {
    if constexpr (HAD) {
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

// Persistent quantizer: CTA c takes the work items c, c + gridDim.x, ... of
// the list (batch * head, block, tensor).  Three tile-sized regions rotate:
// item i's fp16 tile arrives by TMA in region i % 3 (64-channel boxes with
// 128-byte swizzle, chunk c of row t at chunk c ^ (t & 7)) while item i - 1
// is quantized; once item i has read its tile, that region and the free one
// form its fp32 transpose buffer, and when the transpose buffer has been read
// the free region takes item i + 2.
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) quantize_kernel(const __grid_constant__ CUtensorMap map_k,
                                                       const __grid_constant__ CUtensorMap map_v,
                                                       const __grid_constant__ CUtensorMap map_ck,
                                                       const __grid_constant__ CUtensorMap map_cv, QuantArgs a) {
    // INT4 / INT2 code rows leave through a TMA store of a swizzled staging
    // tile (the region just read), so that each warp writes whole lines
    constexpr bool kTmaStore = (BITS == 4 && D * BITS / 8 == 64) || (BITS == 2 && D * BITS / 8 == 32);
    extern __shared__ uint8_t smem_raw[];
    const int t = threadIdx.x;
    uint64_t* bar;  // [3]
    uint8_t* regions;
    QuantSmem<D> sm = carve_quant_smem<D>(smem_raw, bar, regions);
    constexpr uint32_t kTileBytes = quant_region_bytes<D>();
    const int nblk = a.ntok / kT;
    const int nitems = nblk * a.bh * 2;  // < 2^31, checked on the host

    if (t == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
    }
    load_signs<D, HAD>(a, sm, t);
    __syncthreads();
    // item w: tensor w & 1, block (w >> 1) % nblk, batch * head (w >> 1) / nblk
    auto issue = [&](int w, int reg) {
        const int tensor = w & 1;
        const int r = w >> 1;
        const int bh = r / nblk, blk = r - bh * nblk;
        uint8_t* tile = regions + reg * kTileBytes;
        mbar_expect_tx(&bar[reg], kTileBytes);
        const int row0 = bh * a.ntok + blk * kT;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            if (tensor == 0) tma_load_2d(tile + h * (kT * 128), &map_k, h * 64, row0, &bar[reg]);
            else tma_load_2d(tile + h * (kT * 128), &map_v, h * 64, row0, &bar[reg]);
        }
    };
    const int stride = gridDim.x;
    int w = blockIdx.x;
    if (t == 0) {
        if (w < nitems) issue(w, 0);
        if (w + stride < nitems) issue(w + stride, 1);
    }
    int it = 0;
    uint32_t phases = 0;  // bit k: parity of the next completion of region k
    for (; w < nitems; w += stride, ++it) {
        const int reg = it % 3;
        const bool landed = mbar_wait(&bar[reg], (phases >> reg) & 1, 1u << 24);
        if (kTmaStore && t == 0) bulk_wait_read();  // the last code store has read its staging tile
        if (__syncthreads_or(!landed)) {
            if (t == 0) report_error(kErrTmaTimeout);
            break;
        }
        phases ^= 1u << reg;
        const uint8_t* tile = regions + reg * kTileBytes;
        const int spare = (it + 2) % 3;
        sm.tile = tile;
        sm.red_lo = reinterpret_cast<float*>(regions + reg * kTileBytes);
        sm.red_hi = reinterpret_cast<float*>(regions + spare * kTileBytes);
        const int tensor = w & 1;
        const int r = w >> 1;
        const int bh = r / nblk, blk = r - bh * nblk;
        // row t as pairs (channel j, channel j + D/2)
        f2_t P[D / 2];
#pragma unroll
        for (int q = 0; q < D / 16; ++q) {
            const int cl = 8 * q, ch = D / 2 + 8 * q;
            const uint8_t* rl = tile + (cl / 64) * (kT * 128) + t * 128;
            const uint8_t* rh = tile + (ch / 64) * (kT * 128) + t * 128;
            const uint4 lo = *reinterpret_cast<const uint4*>(rl + ((((cl % 64) / 8) ^ (t & 7)) << 4));
            const uint4 hi = *reinterpret_cast<const uint4*>(rh + ((((ch % 64) / 8) ^ (t & 7)) << 4));
            widen_chunk<D, HAD>(lo, hi, q, sm, P);
        }
        if constexpr (MODE != kNsn) __syncthreads();  // the tile region becomes transpose buffer
        const int wn = w + 2 * stride;
        QuantOut out = quant_out<D, BITS, MODE, HAD>(a, tensor, bh, a.blk0 + blk);
        if constexpr (kTmaStore) out.stage = regions + reg * kTileBytes;
        quantize_rows<D, BITS, MODE, HAD>(P, t, sm, out, a.rsqd, a.sqd, [&] {
            if (t == 0 && wn < nitems) {
                fence_proxy_async_smem();
                issue(wn, spare);
            }
        });
        __syncthreads();  // the next item's row loads reuse the shared vectors; codes staged
        if (kTmaStore && t == 0) {
            tma_store_2d(tensor ? &map_cv : &map_ck, 0, bh * a.cap + (a.blk0 + blk) * kT, out.stage);
            bulk_commit();
        }
    }
    if (kTmaStore && t == 0) bulk_wait_read();
    // after an early exit, the copies still in flight (items w and w + stride)
    // land before the CTA ends
    if (t == 0 && w < nitems) {
        for (int k = 0; k < 2; ++k) {
            const int reg = (it + k) % 3;
            if (w + k * stride < nitems) mbar_wait(&bar[reg], (phases >> reg) & 1, 1u << 24);
        }
    }
}

struct AppendArgs {
    QuantArgs q;
    __half* resid[2];
    const __half* x_new[2];  // [B*H][D]
    int slot;                // residual slot of the new token
    int blk;                 // destination block when the slot is the last one
};

// One CTA per (batch*head, tensor).  The new token goes to its residual slot;
// when that slot is the block's last, the CTA instead quantizes the 127 held
// tokens plus the new one into block `blk` (same arithmetic as
// quantize_kernel).
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) append_kernel(AppendArgs a) {
    const int t = threadIdx.x;
    const int bh = blockIdx.x, tensor = blockIdx.y;
    const __half* xn = (tensor ? a.x_new[1] : a.x_new[0]) + (size_t)bh * D;
    __half* res = (tensor ? a.resid[1] : a.resid[0]) + (size_t)bh * kT * D;
    if (a.slot < kT - 1) {
        if (t < D / 8)
            reinterpret_cast<uint4*>(res + (size_t)a.slot * D)[t] = reinterpret_cast<const uint4*>(xn)[t];
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    uint64_t* bar;
    uint8_t* tile;
    QuantSmem<D> sm = carve_quant_smem<D>(smem_raw, bar, tile);
    load_signs<D, HAD>(a.q, sm, t);
    __syncthreads();
    const __half* src = (t == kT - 1) ? xn : res + (size_t)t * D;
    f2_t P[D / 2];
#pragma unroll
    for (int q = 0; q < D / 16; ++q) {
        const uint4 lo = reinterpret_cast<const uint4*>(src)[q];
        const uint4 hi = reinterpret_cast<const uint4*>(src)[D / 16 + q];
        if constexpr (MODE == kNsn) {
            // the fp16 tile in the quantize kernel's layout, for the block means
            const int cl = 8 * q, ch = D / 2 + 8 * q;
            *reinterpret_cast<uint4*>(tile + (cl / 64) * (kT * 128) + t * 128 + ((((cl % 64) / 8) ^ (t & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(tile + (ch / 64) * (kT * 128) + t * 128 + ((((ch % 64) / 8) ^ (t & 7)) << 4)) = hi;
        }
        widen_chunk<D, HAD>(lo, hi, q, sm, P);
    }
    const QuantOut out = quant_out<D, BITS, MODE, HAD>(a.q, tensor, bh, a.blk);
    quantize_rows<D, BITS, MODE, HAD>(P, t, sm, out, a.q.rsqd, a.q.sqd, [] {});
}

struct DequantArgs {
    const uint8_t* codes;
    int pairv;  // V codes of head dim 128: pair-interleaved rows
    const __half* tok;
    const __half* chan;
    const __half* off;
    const int8_t* signs;
    float* out;      // [B*H][ntok][D]
    int cap, ntok, blk0;
    float rsqd, sqd;
};

// One CTA = one block of one (batch, head); thread t rebuilds token t:
//   w = q * sigma; nsep x = n * w, or s (.) (H w * (n rsqd)) under HADAMARD;
//   naive x = w; NSN x = s1 * (b + o) with b = w * (s2 sqd), or
//   s (.) (H w * s2) under HADAMARD.
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) dequantize_kernel(DequantArgs a) {
    using L = RowLayout<D, BITS>;
    const int t = threadIdx.x;
    const int blk = a.blk0 + blockIdx.x, bh = blockIdx.y;
    const int nb = a.cap / kT;
    const int ntk = (MODE == kNsn) ? 2 : 1;
    __shared__ float s_sig[D], s_off[D];
    __shared__ uint32_t s_sgn[D];
    if (t < D) {
        if (MODE != kNaive) s_sig[t] = __half2float(a.chan[((size_t)bh * nb + blk) * D + t]);
        if (MODE == kNsn) s_off[t] = __half2float(a.off[((size_t)bh * nb + blk) * D + t]);
        s_sgn[t] = (HAD && a.signs != nullptr && a.signs[t] < 0) ? 0x80000000u : 0u;
    }
    __syncthreads();
    const size_t tok_idx = (size_t)bh * a.cap + (size_t)blk * kT + t;
    uint32_t w32[L::kWords];
    if (pairv_layout<D>() && a.pairv) {
        // unit u of row t: word u of pair block t / 2, half t & 1
        const uint8_t* pb = a.codes + ((size_t)bh * a.cap + (size_t)blk * kT + (t & ~1)) * L::kBytes;
        const int k = t >> 1;
#pragma unroll
        for (int j = 0; j < L::kWords; ++j) {
            uint32_t h[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int u = 2 * j + e;
                const int c = (u >> 2) ^ pairv_chunk_xor<BITS>(k);
                h[e] = *reinterpret_cast<const uint16_t*>(pb + 16 * c + 4 * (u & 3) + 2 * (t & 1));
            }
            w32[j] = h[0] | (h[1] << 16);
        }
    } else {
        load_words<L::kWords>(a.codes + tok_idx * L::kBytes, w32);
    }
    const __half* tp = a.tok + tok_idx * ntk;
    float w[D];
    const float tsig = (MODE == kNaive) ? __half2float(tp[0]) : 0.0f;
#pragma unroll
    for (int c = 0; c < D; ++c) {
        const float q = (float)((int)code_at<D, BITS>(w32, c) - L::kOff);
        w[c] = __fmul_rn(q, (MODE == kNaive) ? tsig : s_sig[c]);
    }
    if constexpr (HAD) fwht_reg<D>(w);
    float* o = a.out + ((size_t)bh * a.ntok + (size_t)blockIdx.x * kT + t) * D;
    if constexpr (MODE == kNsn) {
        const float s1 = __half2float(tp[0]), s2 = __half2float(tp[1]);
        const float kb = HAD ? s2 : __fmul_rn(s2, a.sqd);
#pragma unroll
        for (int c = 0; c < D; ++c) {
            float b = __fmul_rn(w[c], kb);
            if (HAD) b = __uint_as_float(__float_as_uint(b) ^ s_sgn[c]);
            w[c] = __fmul_rn(s1, __fadd_rn(b, s_off[c]));
        }
    } else if constexpr (MODE == kNsep) {
        const float n = __half2float(tp[0]);
        if constexpr (HAD) {
            const float kd = __fmul_rn(n, a.rsqd);
#pragma unroll
            for (int c = 0; c < D; ++c) w[c] = __uint_as_float(__float_as_uint(__fmul_rn(w[c], kd)) ^ s_sgn[c]);
        } else {
#pragma unroll
            for (int c = 0; c < D; ++c) w[c] = __fmul_rn(n, w[c]);
        }
    }
#pragma unroll
    for (int k = 0; k < D / 4; ++k)
        reinterpret_cast<float4*>(o)[k] = make_float4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
}

}  // namespace kvq
