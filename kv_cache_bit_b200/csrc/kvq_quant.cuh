// kvq_quant.cuh -- block quantizer, residual append/flush and dequantizer
// kernels (sm_100a).  Included once, by kvq_api.cu.
#pragma once

#include "kvq_quant_rows.cuh"

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

// Shared memory of a quantizer CTA: tile-sized regions (128 x D x 2
// bytes; a region also stages a tile's codes for the TMA store once the tile
// has been read), the small vectors and one mbarrier per region.  NSN uses
// three regions: two of them hold the block's fp32 rows for the means (the
// transposed buffer) while the third receives the next tile.
template <int MODE>
__host__ __device__ constexpr int quant_regions() {
    return (is_nsn(MODE) && !kNsnTileMeans) ? 3 : 2;
}

template <int D>
__host__ __device__ constexpr int quant_region_bytes() {
    return kT * D * 2;
}

template <int D, int MODE>
__host__ __device__ constexpr int quant_smem_bytes() {
    // 1024 B alignment slack + regions + vec + group partials + token vector + sign masks + mbarriers
    return 1024 + quant_regions<MODE>() * quant_region_bytes<D>() + D * 4 + kGpartBytes + kT * 4 + D * 4 +
           quant_regions<MODE>() * 8 + 64;
}

// Resident quantizer CTAs per SM the register budget is set for: a thread
// holds a whole row of D fp32 values.  Under NSN that row stays live
// through the block means as well, and the rotated INT3 codes need more
// registers than three CTAs leave; those run two CTAs per SM.
template <int D, int BITS, int MODE, bool HAD>
__host__ __device__ constexpr int quant_min_ctas() {
    return D == 128 ? (((is_nsn(MODE) && !kNsnTileMeans) || (HAD && BITS == 3)) ? 2 : 3) : 4;
}

template <int D, int MODE>
__device__ __forceinline__ QuantSmem<D> carve_quant_smem(uint8_t* base, uint64_t*& bar, uint8_t*& regions) {
    // 1024-byte alignment (TMA 128-byte swizzle) by an offset from the base,
    // so that the pointers stay known to address shared memory
    uint8_t* p = base + ((1024u - (smem_u32(base) & 1023u)) & 1023u);
    QuantSmem<D> sm;
    regions = p;
    sm.tile = p;
    sm.red_lo = reinterpret_cast<float*>(p);
    sm.red_hi = reinterpret_cast<float*>(p + quant_region_bytes<D>());
    p += quant_regions<MODE>() * quant_region_bytes<D>();
    sm.vec = reinterpret_cast<float*>(p);
    p += D * 4;
    sm.gpart = reinterpret_cast<float*>(p);
    p += kGpartBytes;
    sm.tokv = reinterpret_cast<float*>(p);
    p += kT * 4;
    sm.sgn2 = reinterpret_cast<uint32_t*>(p);
    p += D * 4;
    bar = reinterpret_cast<uint64_t*>(p);
    p += quant_regions<MODE>() * 8;
    sm.out = reinterpret_cast<QuantOut*>(p);
    return sm;
}

template <int D, int BITS, int MODE, bool HAD>
__device__ __forceinline__ QuantOut quant_out(const QuantArgs& a, int tensor, int bh, int blk) {
    using L = RowLayout<D, BITS>;
    const int ntk = tok_params(MODE);
    const int nb = a.cap / kT;
    QuantOut o;
    // select with ternaries: a runtime index into the parameter arrays would
    // copy them to local memory
    const bool v = tensor != 0;
    o.codes = (v ? a.codes[1] : a.codes[0]) + ((size_t)bh * a.cap + (size_t)blk * kT) * L::kBytes;
    o.tok = (v ? a.tok[1] : a.tok[0]) + ((size_t)bh * a.cap + (size_t)blk * kT) * ntk;
    o.chan = (MODE != kNaive) ? (v ? a.chan[1] : a.chan[0]) + ((size_t)bh * nb + blk) * D : nullptr;
    o.off = is_nsn(MODE) ? (v ? a.off[1] : a.off[0]) + ((size_t)bh * nb + blk) * off_words<D, MODE>() : nullptr;
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

// Row t of the tile as its raw fp16 chunks (chunk q = channels 8q .. 8q + 7).
template <int D>
__device__ __forceinline__ void load_tile_raw(const uint8_t* tile, int t, uint4 (&raw)[D / 8]) {
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
        const int c = 8 * q;
        raw[q] = *reinterpret_cast<const uint4*>(tile + (c / 64) * (kT * 128) + t * 128 + ((((c % 64) / 8) ^ (t & 7)) << 4));
    }
}

// Persistent quantizer: CTA c takes the work items c, c + gridDim.x, ... of
// the list (batch * head, block, tensor).  NR = quant_regions regions
// rotate: item i's fp16 tile arrives by TMA in region i % NR (64-channel
// boxes with 128-byte swizzle, chunk c of row t at chunk c ^ (t & 7)) while
// earlier items are quantized, and once its rows have been read the region
// stages item i's codes for a TMA store.  With two regions, region (i + 1)
// % 2 takes item i + 2 at the start of item i + 1 (when the store has read
// the staging tile).  With three (NSN), regions i % 3 and (i + 2) % 3 hold
// the block's fp32 rows for the means, after which region (i + 2) % 3 takes
// item i + 2.  A thread owns one token row (D fp32 values in registers),
// and the register budget is set for quant_min_ctas resident CTAs per SM.
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128, (quant_min_ctas<D, BITS, MODE, HAD>())) quantize_kernel(
    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
    const __grid_constant__ CUtensorMap map_ck, const __grid_constant__ CUtensorMap map_cv, QuantArgs a) {
    // INT4 / INT2 code rows leave through a TMA store of a swizzled staging
    // tile (the region just read), so that each warp writes whole lines
    constexpr bool kTmaStore = (BITS == 4 && D * BITS / 8 == 64) || (BITS == 2 && D * BITS / 8 == 32);
    constexpr int NR = quant_regions<MODE>();
    extern __shared__ uint8_t smem_raw[];
    const int t = threadIdx.x;
    uint64_t* bar;  // [NR]
    uint8_t* regions;
    QuantSmem<D> sm = carve_quant_smem<D, MODE>(smem_raw, bar, regions);
    constexpr uint32_t kTileBytes = quant_region_bytes<D>();
    const int nblk = a.ntok / kT;
    const int nitems = nblk * a.bh * 2;  // < 2^31, checked on the host
    const bool signs = HAD && a.signs != nullptr;

    if (t == 0) {
        for (int i = 0; i < NR; ++i) mbar_init(&bar[i], 1);
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
        const int reg = it % NR;
        if (NR == 2 && it > 0 && t == 0) {
            // the previous item's region: free once its code store has read
            // the staging tile; it takes the next item
            if (kTmaStore) bulk_wait_read();
            if (w + stride < nitems) {
                fence_proxy_async_smem();
                issue(w + stride, reg ^ 1);
            }
        }
        if (t == 0) {
            // the item's output pointers, published by the barrier below (the
            // threads read them from shared memory where they are used)
            const int r = w >> 1;
            const int bh = r / nblk, blk = r - bh * nblk;
            QuantOut o = quant_out<D, BITS, MODE, HAD>(a, w & 1, bh, a.blk0 + blk);
            if constexpr (kTmaStore) o.stage = regions + reg * kTileBytes;
            *sm.out = o;
        }
        const bool landed = mbar_wait(&bar[reg], (phases >> reg) & 1, KVQ_WAIT_LIMIT(1u << 24));
        if (__syncthreads_or(!landed)) {
            if (t == 0) report_error(kErrTmaTimeout);
            break;
        }
        phases ^= 1u << reg;
        uint8_t* tile = regions + reg * kTileBytes;
        sm.tile = tile;
        const int spare = (reg + 2) % NR;  // NSN: the region of the item after next
        sm.red_lo = reinterpret_cast<float*>(tile);
        sm.red_hi = reinterpret_cast<float*>(regions + spare * kTileBytes);
        const int tensor = w & 1;
        const int r = w >> 1;
        const int bh = r / nblk, blk = r - bh * nblk;
        uint4 raw[D / 8];
        load_tile_raw<D>(tile, t, raw);
        const QuantOut& out = *sm.out;
        // NSN: the spare region is written once the previous item's code store
        // has read it, and takes item w + 2 stride after the means
        auto before_spill = [&] {
            if (NR == 3 && kTmaStore && t == 0) bulk_wait_read();
        };
        auto after_means = [&] {
            if (NR == 3 && t == 0 && w + 2 * stride < nitems) {
                fence_proxy_async_smem();
                issue(w + 2 * stride, spare);
            }
        };
        if (signs) quantize_rows<D, BITS, MODE, HAD, true>(raw, t, sm, out, a.rsqd, a.sqd, before_spill, after_means);
        else quantize_rows<D, BITS, MODE, HAD, false>(raw, t, sm, out, a.rsqd, a.sqd, before_spill, after_means);
        __syncthreads();  // codes staged; the next item's rows reuse the shared vectors
        if (kTmaStore && t == 0) {
            tma_store_2d(tensor ? &map_cv : &map_ck, 0, bh * a.cap + (a.blk0 + blk) * kT, tile);
            bulk_commit();
        }
    }
    if (kTmaStore && t == 0) bulk_wait_read();
    // after an early exit, the copies still in flight land before the CTA
    // ends: items w and w + stride (both issued by then), and under NSN item
    // w + 2 stride when item w - stride issued it
    if (t == 0 && w < nitems) {
        for (int k = 0; k < NR; ++k) {
            const int reg = (it + k) % NR;
            const bool issued = k < 2 || it > 0;
            if (issued && w + k * stride < nitems) mbar_wait(&bar[reg], (phases >> reg) & 1, 1u << 24);
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

// The new token of every (batch*head, tensor) into its residual slot, when
// that slot is not the block's last: one 16-byte chunk per thread.  The
// decode kernel behind it may be scheduled at once.
template <int D>
__global__ void __launch_bounds__(256) append_copy_kernel(AppendArgs a, int bh) {
    grid_dep_launch();
    constexpr int NC = D / 8;  // 16-byte chunks per row
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= 2 * bh * NC) return;
    const int tensor = i / (bh * NC), r = i - tensor * bh * NC, row = r / NC, c = r - row * NC;
    const uint4* src = reinterpret_cast<const uint4*>((tensor ? a.x_new[1] : a.x_new[0]) + (size_t)row * D) + c;
    uint4* dst = reinterpret_cast<uint4*>((tensor ? a.resid[1] : a.resid[0]) + ((size_t)row * kT + a.slot) * D) + c;
    *dst = *src;
}

// One CTA per (batch*head, tensor), launched when the new token's slot is
// the block's last: the CTA quantizes the 127 held tokens plus the new one
// into block `blk` (same arithmetic as quantize_kernel).
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) append_kernel(AppendArgs a) {
    const int t = threadIdx.x;
    const int bh = blockIdx.x, tensor = blockIdx.y;
    const __half* xn = (tensor ? a.x_new[1] : a.x_new[0]) + (size_t)bh * D;
    __half* res = (tensor ? a.resid[1] : a.resid[0]) + (size_t)bh * kT * D;
    extern __shared__ uint8_t smem_raw[];
    uint64_t* bar;
    uint8_t* regions;
    QuantSmem<D> sm = carve_quant_smem<D, MODE>(smem_raw, bar, regions);
    load_signs<D, HAD>(a.q, sm, t);
    __syncthreads();
    const __half* src = (t == kT - 1) ? xn : res + (size_t)t * D;
    uint4 raw[D / 8];
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
        raw[q] = reinterpret_cast<const uint4*>(src)[q];
        if constexpr (is_nsn(MODE) && kNsnTileMeans) {
            // the fp16 tile in the quantize kernel's layout, for the block means
            const int c = 8 * q;
            *reinterpret_cast<uint4*>(regions + (c / 64) * (kT * 128) + t * 128 + ((((c % 64) / 8) ^ (t & 7)) << 4)) =
                raw[q];
        }
    }
    if (t == 0) *sm.out = quant_out<D, BITS, MODE, HAD>(a.q, tensor, bh, a.blk);
    __syncthreads();
    const QuantOut& out = *sm.out;
    auto none = [] {};
    if (HAD && a.q.signs != nullptr)
        quantize_rows<D, BITS, MODE, HAD, true>(raw, t, sm, out, a.q.rsqd, a.q.sqd, none, none);
    else
        quantize_rows<D, BITS, MODE, HAD, false>(raw, t, sm, out, a.q.rsqd, a.q.sqd, none, none);
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

// Token row rebuilt in fp32 from its code words w32 and parameters (tp: its
// per-token fp16 values; s1dq: its s1 rebuilt from the block record under
// DQ; sig, off: the block's channel scales and means as fp32; sgn: the
// rotation's signs as fp32 sign-bit masks), in the oracle's operation order:
//   w = q * sigma; nsep x = n * w, or s (.) (H w * (n rsqd)) under HADAMARD;
//   naive x = w; NSN x = s1 * (b + o) with b = w * (s2 sqd), or
//   s (.) (H w * s2) under HADAMARD.
template <int D, int BITS, int MODE, bool HAD>
__device__ __forceinline__ void dequant_row(const uint32_t (&w32)[RowLayout<D, BITS>::kWords], const __half* tp,
                                            float s1dq, const float* sig, const float* off, const uint32_t* sgn,
                                            float rsqd, float sqd, float (&w)[D]) {
    using L = RowLayout<D, BITS>;
    const float tsig = (MODE == kNaive) ? __half2float(tp[0]) : 0.0f;
#pragma unroll
    for (int c = 0; c < D; ++c) {
        const float q = (float)((int)code_at<D, BITS>(w32, c) - L::kOff);
        w[c] = __fmul_rn(q, (MODE == kNaive) ? tsig : sig[c]);
    }
    if constexpr (HAD) fwht_reg<D>(w);
    if constexpr (is_nsn(MODE)) {
        // under DQ s1 comes from the block record (s1dq) and tp holds s2 only
        const float s1 = (MODE == kNsnDq) ? s1dq : __half2float(tp[0]);
        const float s2 = __half2float(tp[MODE == kNsnDq ? 0 : 1]);
        const float kb = HAD ? s2 : __fmul_rn(s2, sqd);
#pragma unroll
        for (int c = 0; c < D; ++c) {
            float b = __fmul_rn(w[c], kb);
            if (HAD) b = __uint_as_float(__float_as_uint(b) ^ sgn[c]);
            w[c] = __fmul_rn(s1, __fadd_rn(b, off[c]));
        }
    } else if constexpr (MODE == kNsep) {
        const float n = __half2float(tp[0]);
        if constexpr (HAD) {
            const float kd = __fmul_rn(n, rsqd);
#pragma unroll
            for (int c = 0; c < D; ++c) w[c] = __uint_as_float(__float_as_uint(__fmul_rn(w[c], kd)) ^ sgn[c]);
        } else {
#pragma unroll
            for (int c = 0; c < D; ++c) w[c] = __fmul_rn(n, w[c]);
        }
    }
}

// One CTA = one block of one (batch, head); thread t rebuilds token t.
template <int D, int BITS, int MODE, bool HAD>
__global__ void __launch_bounds__(128) dequantize_kernel(DequantArgs a) {
    using L = RowLayout<D, BITS>;
    const int t = threadIdx.x;
    const int blk = a.blk0 + blockIdx.x, bh = blockIdx.y;
    const int nb = a.cap / kT;
    const int ntk = tok_params(MODE);
    __shared__ float s_sig[D], s_off[D];
    __shared__ uint32_t s_sgn[D];
    const __half* offb = is_nsn(MODE) ? a.off + ((size_t)bh * nb + blk) * off_words<D, MODE>() : nullptr;
    float s1dq = 0.0f;
    if constexpr (MODE == kNsnDq) s1dq = dq_s1<D>(reinterpret_cast<const uint8_t*>(offb), t);
    if (t < D) {
        if (MODE != kNaive) s_sig[t] = __half2float(a.chan[((size_t)bh * nb + blk) * D + t]);
        if (MODE == kNsn) s_off[t] = __half2float(offb[t]);
        if (MODE == kNsnDq) s_off[t] = dq_o<D>(reinterpret_cast<const uint8_t*>(offb), t);
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
    float w[D];
    dequant_row<D, BITS, MODE, HAD>(w32, a.tok + tok_idx * ntk, s1dq, s_sig, s_off, s_sgn, a.rsqd, a.sqd, w);
    float* o = a.out + ((size_t)bh * a.ntok + (size_t)blockIdx.x * kT + t) * D;
#pragma unroll
    for (int k = 0; k < D / 4; ++k)
        reinterpret_cast<float4*>(o)[k] = make_float4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
}

// ---------------------------------------------------------------- sign selection

struct SelectArgs {
    const __half* x;      // [n_blocks][128][D] the sample
    const int8_t* signs;  // [n_cand][D] candidate sign vectors
    double* part;         // [n_cand][n_blocks] error of each (candidate, block)
    int n_blocks;
    float rsqd, sqd;
};

// Pairwise (recursive halving) fp64 sum of the squared differences between
// the rebuilt row w and the input row x over channels [OFF, OFF + N).
template <int OFF, int N, int D>
__device__ __forceinline__ double row_sq_err(const float (&w)[D], const __half* x) {
    if constexpr (N == 1) {
        const double df = __dsub_rn((double)w[OFF], (double)__half2float(x[OFF]));
        return __dmul_rn(df, df);
    } else {
        return __dadd_rn(row_sq_err<OFF, N / 2, D>(w, x), row_sq_err<OFF + N / 2, N / 2, D>(w, x));
    }
}

static_assert(dq_record_bytes<64>() <= 64 * 2 && dq_record_bytes<128>() <= 128 * 2,
              "a block record fits the means buffer of the selection kernel");

template <int D, int BITS, int MODE>
__host__ __device__ constexpr int select_smem_bytes() {
    // the quantizer's scratch, then the block's outputs and the per-row errors
    return (quant_smem_bytes<D, MODE>() + 127) / 128 * 128 + kT * RowLayout<D, BITS>::kBytes + kT * 2 * 2 +
           D * 2 * 2 + D * 4 * 3 + kT * 8;
}

// CTA (block b, candidate k): the block quantized with candidate k's signs
// exactly as the quantize kernel does, rebuilt as dequantize does, and the
// block's reconstruction error: per row the pairwise sum over channels of
// (x_hat - x)^2 in fp64, over the rows the pairwise sum over tokens.
template <int D, int BITS, int MODE>
__global__ void __launch_bounds__(128) select_signs_kernel(SelectArgs a) {
    using L = RowLayout<D, BITS>;
    constexpr int ntk = tok_params(MODE);
    const int t = threadIdx.x, blk = blockIdx.x, cand = blockIdx.y;
    extern __shared__ uint8_t smem_raw[];
    uint64_t* bar;
    uint8_t* regions;
    QuantSmem<D> sm = carve_quant_smem<D, MODE>(smem_raw, bar, regions);
    uint8_t* p = smem_raw + (quant_smem_bytes<D, MODE>() + 127) / 128 * 128;
    uint8_t* s_codes = p;                                    p += kT * L::kBytes;
    __half* s_tok = reinterpret_cast<__half*>(p);            p += kT * 2 * 2;
    __half* s_chan = reinterpret_cast<__half*>(p);           p += D * 2;
    __half* s_off16 = reinterpret_cast<__half*>(p);          p += D * 2;
    float* s_sig = reinterpret_cast<float*>(p);              p += D * 4;
    float* s_off = reinterpret_cast<float*>(p);              p += D * 4;
    uint32_t* s_sgn = reinterpret_cast<uint32_t*>(p);        p += D * 4;
    double* s_err = reinterpret_cast<double*>(p);
    const int8_t* sg = a.signs + (size_t)cand * D;
    if (t < D / 2) sm.sgn2[t] = (sg[2 * t] < 0 ? 0x8000u : 0u) | (sg[2 * t + 1] < 0 ? 0x80000000u : 0u);
    if (t < D) s_sgn[t] = sg[t] < 0 ? 0x80000000u : 0u;
    __syncthreads();
    const __half* xr = a.x + ((size_t)blk * kT + t) * D;
    uint4 raw[D / 8];
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
        raw[q] = reinterpret_cast<const uint4*>(xr)[q];
        if constexpr (is_nsn(MODE) && kNsnTileMeans) {
            // the fp16 tile in the quantize kernel's layout, for the block means
            const int c = 8 * q;
            *reinterpret_cast<uint4*>(regions + (c / 64) * (kT * 128) + t * 128 + ((((c % 64) / 8) ^ (t & 7)) << 4)) =
                raw[q];
        }
    }
    if (t == 0) {
        QuantOut o;
        o.codes = s_codes;
        o.stage = nullptr;
        o.tok = s_tok;
        o.chan = s_chan;
        o.off = s_off16;
        o.pairv = false;
        *sm.out = o;
    }
    __syncthreads();
    const QuantOut& out = *sm.out;
    auto none = [] {};
    quantize_rows<D, BITS, MODE, true, true>(raw, t, sm, out, a.rsqd, a.sqd, none, none);
    __syncthreads();
    if (t < D) {
        s_sig[t] = __half2float(s_chan[t]);
        s_off[t] = (MODE == kNsn) ? __half2float(s_off16[t])
                 : (MODE == kNsnDq) ? dq_o<D>(reinterpret_cast<const uint8_t*>(s_off16), t) : 0.0f;
    }
    __syncthreads();
    uint32_t w32[L::kWords];
    load_words<L::kWords>(s_codes + (size_t)t * L::kBytes, w32);
    float w[D];
    const float s1dq = (MODE == kNsnDq) ? dq_s1<D>(reinterpret_cast<const uint8_t*>(s_off16), t) : 0.0f;
    dequant_row<D, BITS, MODE, true>(w32, s_tok + t * ntk, s1dq, s_sig, s_off, s_sgn, a.rsqd, a.sqd, w);
    s_err[t] = row_sq_err<0, D, D>(w, xr);
    __syncthreads();
#pragma unroll
    for (int h = 1; h < kT; h *= 2) {
        if ((t & (2 * h - 1)) == 0) s_err[t] = __dadd_rn(s_err[t], s_err[t + h]);
        __syncthreads();
    }
    if (t == 0) a.part[(size_t)cand * a.n_blocks + blk] = s_err[0];
}

// Errors of the candidates (their blocks added in order) and the index of
// the smallest one (the lowest index among equal ones).
__global__ void __launch_bounds__(256) select_reduce_kernel(const double* part, int n_blocks, int n_cand,
                                                            double* err, int* best) {
    __shared__ double s_e[256];
    const int k = threadIdx.x;
    if (k < n_cand) {
        double e = 0.0;
        for (int b = 0; b < n_blocks; ++b) e = __dadd_rn(e, part[(size_t)k * n_blocks + b]);
        err[k] = e;
        s_e[k] = e;
    }
    __syncthreads();
    if (k == 0) {
        int bi = 0;
        for (int j = 1; j < n_cand; ++j)
            if (s_e[j] < s_e[bi]) bi = j;
        *best = bi;
    }
}

}  // namespace kvq
