// kvq_api.cu -- host side of libkvq: argument checks, shape arithmetic,
// tensor-map set-up and kernel launches behind the C ABI of include/kvq.h.
// This is the library's single translation unit; the kernels come in from
// the .cuh files below.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "kvq.h"
#include "kvq_decode_mma.cuh"
#include "kvq_decode_simple.cuh"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around each entry point (no cost beyond a few loads unless
// a profiler has attached its NVTX hooks).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

struct ModeInfo {
    int mode = -1;
    bool had = false;
};

ModeInfo mode_of(uint32_t flags) {
    ModeInfo m;
    const uint32_t base = flags & ~uint32_t(KVQ_HADAMARD);
    m.had = (flags & KVQ_HADAMARD) != 0;
    if (base == (KVQ_NORM_SEP | KVQ_PER_CHANNEL)) m.mode = kNsep;
    else if (flags == 0) m.mode = kNaive;
    else if (base == (KVQ_NSN | KVQ_PER_CHANNEL)) m.mode = kNsn;
    else if (base == (KVQ_NSN | KVQ_PER_CHANNEL | KVQ_DQ)) m.mode = kNsnDq;
    return m;
}

int off_words_of(int mode, int d) {
    if (!is_nsn(mode)) return 0;
    if (mode == kNsn) return d;
    return d == 64 ? off_words<64, kNsnDq>() : off_words<128, kNsnDq>();
}

int row_bytes(int d, int bits) {
    if ((d != 64 && d != 128) || bits < 2 || bits > 4) return 0;
    return d * bits / 8;
}

// Status of a config; fills mode info.
kvq_status check_cfg(const kvq_config* cfg, ModeInfo* mi) {
    if (cfg == nullptr) return KVQ_ERR_INVALID_ARG;
    if (cfg->reserved != 0) return KVQ_ERR_INVALID_ARG;
    if (cfg->signs != nullptr && !aligned16(cfg->signs)) return KVQ_ERR_INVALID_ARG;
    if (row_bytes(cfg->head_dim, cfg->bits) == 0) return KVQ_ERR_UNSUPPORTED;
    *mi = mode_of(cfg->flags);
    if (mi->mode < 0) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

// Shape and pointer checks of a cache against a config.
kvq_status check_cache(const kvq_config* cfg, const ModeInfo& mi, const kvq_cache* c) {
    if (c == nullptr) return KVQ_ERR_INVALID_ARG;
    if (c->batch < 1 || c->kv_heads < 1 || c->head_dim != cfg->head_dim) return KVQ_ERR_INVALID_ARG;
    if (c->capacity < kT || c->capacity % kT != 0) return KVQ_ERR_INVALID_ARG;
    if (c->len < 0 || c->len > c->capacity) return KVQ_ERR_INVALID_ARG;
    if ((int64_t)c->batch * c->kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
    for (int i = 0; i < 2; ++i) {
        if (!ok_ptr(c->codes[i]) || !ok_ptr(c->tok[i]) || !ok_ptr(c->resid[i])) return KVQ_ERR_INVALID_ARG;
        if (mi.mode != kNaive && !ok_ptr(c->chan[i])) return KVQ_ERR_INVALID_ARG;
        if (is_nsn(mi.mode) && !ok_ptr(c->off[i])) return KVQ_ERR_INVALID_ARG;
    }
    return KVQ_OK;
}

kvq_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

float rsqd_of(int d) { return (float)(1.0 / std::sqrt((double)d)); }
float sqd_of(int d) { return (float)std::sqrt((double)d); }

// Compile-time dispatch over (head_dim, bits, mode, hadamard).
template <int D, int BITS, typename Fn>
kvq_status dispatch_mode(const ModeInfo& mi, Fn& fn) {
    if (mi.mode == kNsep) return mi.had ? fn.template run<D, BITS, kNsep, true>() : fn.template run<D, BITS, kNsep, false>();
    if (mi.mode == kNaive) return mi.had ? KVQ_ERR_UNSUPPORTED : fn.template run<D, BITS, kNaive, false>();
    if (mi.mode == kNsnDq) return mi.had ? fn.template run<D, BITS, kNsnDq, true>() : fn.template run<D, BITS, kNsnDq, false>();
    return mi.had ? fn.template run<D, BITS, kNsn, true>() : fn.template run<D, BITS, kNsn, false>();
}

template <typename Fn>
kvq_status dispatch(int d, int bits, const ModeInfo& mi, Fn& fn) {
    if (d == 64) {
        if (bits == 2) return dispatch_mode<64, 2>(mi, fn);
        if (bits == 3) return dispatch_mode<64, 3>(mi, fn);
        if (bits == 4) return dispatch_mode<64, 4>(mi, fn);
    } else if (d == 128) {
        if (bits == 2) return dispatch_mode<128, 2>(mi, fn);
        if (bits == 3) return dispatch_mode<128, 3>(mi, fn);
        if (bits == 4) return dispatch_mode<128, 4>(mi, fn);
    }
    return KVQ_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------- TMA maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D view [rows][d] of fp16 rows; boxes of 64 channels x 128 rows with
// 128-byte swizzle.
bool make_row_map(CUtensorMap* m, const void* base, uint64_t rows, int d) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kT};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view [rows][row_bytes] of packed code rows (row_bytes 64 or 32), as
// the destination of TMA stores of 128-row tiles with the matching swizzle
// (64-byte rows: 64-byte swizzle; 32-byte rows: 32-byte swizzle).
bool make_code_map(CUtensorMap* m, void* base, uint64_t rows, int row_bytes) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)kT};
    cuuint32_t es[2] = {1, 1};
    const CUtensorMapSwizzle sw = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory size, and the largest shared-memory carveout so that
// the residency the occupancy calculator reports is the one the launch gets.
template <typename K>
bool set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
           cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

// set_smem once per (kernel, device): function attributes belong to a
// device's context.  One bit per device id; racing callers both set the same
// attributes, which is harmless.
template <auto Kernel>
bool ensure_smem(int bytes) {
    static std::atomic<uint64_t> done{0};  // one mask per kernel instantiation
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const uint64_t bit = uint64_t(1) << dev;
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (!set_smem(Kernel, bytes)) return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

QuantArgs quant_args(const kvq_config* cfg, const kvq_cache* c) {
    QuantArgs a;
    for (int i = 0; i < 2; ++i) {
        a.codes[i] = c->codes[i];
        a.tok[i] = reinterpret_cast<__half*>(c->tok[i]);
        a.chan[i] = reinterpret_cast<__half*>(c->chan[i]);
        a.off[i] = reinterpret_cast<__half*>(c->off[i]);
    }
    a.signs = cfg->signs;
    a.H = c->kv_heads;
    a.cap = c->capacity;
    a.ntok = 0;
    a.blk0 = 0;
    a.rsqd = rsqd_of(cfg->head_dim);
    a.sqd = sqd_of(cfg->head_dim);
    return a;
}

// ---------------------------------------------------------------- launchers

struct QuantLaunch {
    QuantArgs a;
    const void* k;
    const void* v;
    int bh;
    int nblk;
    cudaStream_t st;
    template <int D, int BITS, int MODE, bool HAD>
    kvq_status run() {
        CUtensorMap mk, mv, mck, mcv;
        const uint64_t rows = (uint64_t)bh * (uint64_t)a.ntok;
        if (!make_row_map(&mk, k, rows, D) || !make_row_map(&mv, v, rows, D)) return KVQ_ERR_CUDA;
        memset(&mck, 0, sizeof(mck));
        memset(&mcv, 0, sizeof(mcv));
        constexpr int rb = D * BITS / 8;
        if constexpr ((BITS == 4 && rb == 64) || (BITS == 2 && rb == 32)) {
            const uint64_t crow = (uint64_t)bh * (uint64_t)a.cap;
            if (crow >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
            if (!make_code_map(&mck, a.codes[0], crow, rb) || !make_code_map(&mcv, a.codes[1], crow, rb))
                return KVQ_ERR_CUDA;
        }
        constexpr int smem = quant_smem_bytes<D, MODE>();
        auto kern = quantize_kernel<D, BITS, MODE, HAD>;
        if (!ensure_smem<quantize_kernel<D, BITS, MODE, HAD>>(smem)) return KVQ_ERR_CUDA;
        int dev = 0, sms = 0, occ = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kT, smem) != cudaSuccess)
            return KVQ_ERR_CUDA;
        const long long items = (long long)nblk * bh * 2;
        if (items >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
        long long grid = (long long)sms * (occ > 0 ? occ : 1);
        if (grid > items) grid = items;
        a.bh = bh;
        kern<<<(unsigned)grid, kT, smem, st>>>(mk, mv, mck, mcv, a);
        return launch_status();
    }
};

struct AppendLaunch {
    AppendArgs a;
    int bh;
    cudaStream_t st;
    template <int D, int BITS, int MODE, bool HAD>
    kvq_status run() {
        if (a.slot < kT - 1) {
            // a plain copy into the residual slot
            const int n = 2 * bh * (D / 8);
            append_copy_kernel<D><<<(n + 255) / 256, 256, 0, st>>>(a, bh);
            return launch_status();
        }
        constexpr int smem = quant_smem_bytes<D, MODE>();
        if (!ensure_smem<append_kernel<D, BITS, MODE, HAD>>(smem)) return KVQ_ERR_CUDA;
        append_kernel<D, BITS, MODE, HAD><<<dim3(bh, 2), kT, smem, st>>>(a);
        return launch_status();
    }
};

struct DequantLaunch {
    DequantArgs a;
    int bh, nblk;
    cudaStream_t st;
    template <int D, int BITS, int MODE, bool HAD>
    kvq_status run() {
        dequantize_kernel<D, BITS, MODE, HAD><<<dim3(nblk, bh), kT, 0, st>>>(a);
        return launch_status();
    }
};

struct SelectLaunch {
    SelectArgs a;
    int n_cand;
    double* err;
    int* best;
    cudaStream_t st;
    template <int D, int BITS, int MODE, bool HAD>
    kvq_status run() {
        if constexpr (!HAD || MODE == kNaive) {
            return KVQ_ERR_UNSUPPORTED;
        } else {
            constexpr int smem = select_smem_bytes<D, BITS, MODE>();
            if (!ensure_smem<select_signs_kernel<D, BITS, MODE>>(smem)) return KVQ_ERR_CUDA;
            select_signs_kernel<D, BITS, MODE><<<dim3(a.n_blocks, n_cand), kT, smem, st>>>(a);
            kvq_status s = launch_status();
            if (s != KVQ_OK) return s;
            select_reduce_kernel<<<1, 256, 0, st>>>(a.part, a.n_blocks, n_cand, err, best);
            return launch_status();
        }
    }
};

template <int D, int BITS, int MODE, bool HAD, int GP>
kvq_status launch_decode_mma(DecodeArgs a, int bh, cudaStream_t st) {
    constexpr int smem = mma_smem_bytes<D, BITS, MODE, GP>();
    auto kern = decode_mma_kernel<D, BITS, MODE, HAD, GP>;
    if (!ensure_smem<decode_mma_kernel<D, BITS, MODE, HAD, GP>>(smem)) return KVQ_ERR_CUDA;
    int dev = 0, sms = 0, occ = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kNW * 32, smem) != cudaSuccess)
        return KVQ_ERR_CUDA;
    int grid = sms * (occ > 0 ? occ : 1);
    if (grid > kMaxCtasPerSM * sms) grid = kMaxCtasPerSM * sms;
    a.nwarps = (long long)grid * kNW;
    a.work = (long long)bh * a.nbq;
    if (a.work >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
    if (a.work > 0) {
        // a programmatic dependent of the kernel ahead of it in the stream:
        // its launch overlaps that kernel's tail (the kernel waits for it
        // before touching memory)
        cudaLaunchConfig_t dc = {};
        dc.gridDim = dim3(grid);
        dc.blockDim = dim3(kNW * 32);
        dc.dynamicSmemBytes = smem;
        dc.stream = st;
        cudaLaunchAttribute da[1];
        da[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        da[0].val.programmaticStreamSerializationAllowed = 1;
        dc.attrs = da;
        dc.numAttrs = 1;
        if (cudaLaunchKernelEx(&dc, kern, a) != cudaSuccess) return KVQ_ERR_CUDA;
        kvq_status s = launch_status();
        if (s != KVQ_OK) return s;
    }
    // the combine kernel is a programmatic dependent of the decode kernel:
    // its residual phase overlaps the decode kernel's tail
    auto comb = decode_combine_mma_kernel<D, GP>;
    constexpr int csmem = combine_smem_bytes<D>();
    if (!ensure_smem<decode_combine_mma_kernel<D, GP>>(csmem)) return KVQ_ERR_CUDA;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(bh);
    lc.blockDim = dim3(128);
    lc.dynamicSmemBytes = csmem;
    lc.stream = st;
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[0].val.programmaticStreamSerializationAllowed = a.work > 0 ? 1 : 0;
    lc.attrs = la;
    lc.numAttrs = 1;
    if (cudaLaunchKernelEx(&lc, comb, a) != cudaSuccess) return KVQ_ERR_CUDA;
    return launch_status();
}

struct DecodeLaunch {
    DecodeArgs a;
    int bh;
    cudaStream_t st;
    template <int D, int BITS, int MODE, bool HAD>
    kvq_status run() {
        if constexpr (D == 128) {
            // tensor-core path
            if (a.G <= 4) return launch_decode_mma<D, BITS, MODE, HAD, 4>(a, bh, st);
            return launch_decode_mma<D, BITS, MODE, HAD, 8>(a, bh, st);
        } else {
            decode_split_kernel<D, BITS, MODE, HAD><<<dim3(a.nsplit, bh), kT, 0, st>>>(a);
            kvq_status s = launch_status();
            if (s != KVQ_OK) return s;
            decode_combine_kernel<D, HAD><<<bh, kT, 0, st>>>(a);
            return launch_status();
        }
    }
};

// Splits of the sequence for the CUDA-core decode (head dim 64): about six
// waves of CTAs on 148 SMs (two resident per SM), at least 8 blocks per
// split when the sequence is long enough to fill the waves that way, else
// as few as one block per split (short caches are latency-bound).  Fixed
// per cache shape so that the workspace size does not depend on len.
int decode_splits(const kvq_cache* c) {
    const int bh = c->batch * c->kv_heads;
    const int nb = c->capacity / kT;
    int ns = (6 * 296 + bh - 1) / bh;
    const int cap8 = nb / 8;
    if (ns > cap8) ns = cap8 >= 2 ? cap8 : nb;
    if (ns < 1) ns = 1;
    return ns;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

int32_t kvq_row_bytes(int32_t head_dim, int32_t bits) { return row_bytes(head_dim, bits); }

int32_t kvq_tok_params(uint32_t flags) {
    const ModeInfo mi = mode_of(flags);
    if (mi.mode < 0 || (mi.mode == kNaive && mi.had)) return -1;
    return tok_params(mi.mode);
}

int32_t kvq_off_words(uint32_t flags, int32_t head_dim) {
    const ModeInfo mi = mode_of(flags);
    if (mi.mode < 0 || (mi.mode == kNaive && mi.had) || (head_dim != 64 && head_dim != 128)) return -1;
    return off_words_of(mi.mode, head_dim);
}

kvq_status kvq_make_signs(uint64_t seed, int32_t head_dim, int8_t* host_out) {
    if (host_out == nullptr || head_dim < 1) return KVQ_ERR_INVALID_ARG;
    uint64_t state = seed;
    for (int32_t c = 0; c < head_dim; ++c) {
        // SplitMix64 step (Steele, Lea & Flood 2014)
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        host_out[c] = (z >> 63) ? int8_t(-1) : int8_t(1);
    }
    return KVQ_OK;
}

kvq_status kvq_quantize_block(const kvq_config* cfg, kvq_cache* cache, const uint16_t* k, const uint16_t* v,
                              int64_t t0, int64_t ntok, void* stream) {
    NvtxRange nvtx_range("kvq_quantize_block");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if ((s = check_cache(cfg, mi, cache)) != KVQ_OK) return s;
    if (!ok_ptr(k) || !ok_ptr(v)) return KVQ_ERR_INVALID_ARG;
    if (t0 < 0 || ntok <= 0 || t0 % kT != 0 || ntok % kT != 0) return KVQ_ERR_INVALID_ARG;
    if (t0 + ntok > cache->capacity) return KVQ_ERR_CAPACITY;
    const int64_t held0 = (cache->len / kT) * kT;
    if (cache->len % kT != 0 && t0 + ntok > held0) return KVQ_ERR_INVALID_ARG;
    const int bh = cache->batch * cache->kv_heads;
    if ((uint64_t)bh * (uint64_t)ntok >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    QuantLaunch L;
    L.a = quant_args(cfg, cache);
    L.a.ntok = (int)ntok;
    L.a.blk0 = (int)(t0 / kT);
    L.k = k;
    L.v = v;
    L.bh = bh;
    L.nblk = (int)(ntok / kT);
    L.st = static_cast<cudaStream_t>(stream);
    if ((s = dispatch(cfg->head_dim, cfg->bits, mi, L)) != KVQ_OK) return s;
    if (t0 + ntok > cache->len) cache->len = t0 + ntok;
    return KVQ_OK;
}

kvq_status kvq_append_token(const kvq_config* cfg, kvq_cache* cache, const uint16_t* k_new, const uint16_t* v_new,
                            void* stream) {
    NvtxRange nvtx_range("kvq_append_token");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if ((s = check_cache(cfg, mi, cache)) != KVQ_OK) return s;
    if (!ok_ptr(k_new) || !ok_ptr(v_new)) return KVQ_ERR_INVALID_ARG;
    if (cache->len + 1 > cache->capacity) return KVQ_ERR_CAPACITY;
    AppendLaunch L;
    L.a.q = quant_args(cfg, cache);
    for (int i = 0; i < 2; ++i) L.a.resid[i] = reinterpret_cast<__half*>(cache->resid[i]);
    L.a.x_new[0] = reinterpret_cast<const __half*>(k_new);
    L.a.x_new[1] = reinterpret_cast<const __half*>(v_new);
    L.a.slot = (int)(cache->len % kT);
    L.a.blk = (int)(cache->len / kT);
    L.bh = cache->batch * cache->kv_heads;
    L.st = static_cast<cudaStream_t>(stream);
    if ((s = dispatch(cfg->head_dim, cfg->bits, mi, L)) != KVQ_OK) return s;
    cache->len += 1;
    return KVQ_OK;
}

size_t kvq_decode_workspace_bytes(const kvq_config* cfg, const kvq_cache* cache, int32_t q_heads) {
    ModeInfo mi;
    if (check_cfg(cfg, &mi) != KVQ_OK || check_cache(cfg, mi, cache) != KVQ_OK) return 0;
    if (q_heads < cache->kv_heads || q_heads % cache->kv_heads != 0) return 0;
    const int G = q_heads / cache->kv_heads;
    if (G > kGMax) return 0;
    const size_t bh = (size_t)cache->batch * cache->kv_heads;
    // tensor-core path: one partial per (warp, pair) segment, kNW slots per
    // (CTA, pair) meeting; those are bounded by (largest persistent grid on
    // the current device) + (pairs)
    if (cfg->head_dim == 128) {
        // without a usable device (host-side checks), the bound of a 256-SM part
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
            cudaGetLastError();
            sms = 256;
        }
        const size_t max_ctas = (size_t)kMaxCtasPerSM * (size_t)sms;
        return (size_t)kNW * (max_ctas + bh) * (size_t)G * part_stride<128>() * sizeof(float);
    }
    return bh * (size_t)decode_splits(cache) * (size_t)G * (2 + 2 * (size_t)cfg->head_dim) * sizeof(float);
}

kvq_status kvq_decode_attention(const kvq_config* cfg, const kvq_cache* cache, const uint16_t* q, int32_t q_heads,
                                float scale, float* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("kvq_decode_attention");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if ((s = check_cache(cfg, mi, cache)) != KVQ_OK) return s;
    if (!ok_ptr(q) || !ok_ptr(out)) return KVQ_ERR_INVALID_ARG;
    if (q_heads < cache->kv_heads || q_heads % cache->kv_heads != 0) return KVQ_ERR_INVALID_ARG;
    const int G = q_heads / cache->kv_heads;
    if (G > kGMax) return KVQ_ERR_UNSUPPORTED;
    const size_t need = kvq_decode_workspace_bytes(cfg, cache, q_heads);
    if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return KVQ_ERR_WORKSPACE;
    DecodeLaunch L;
    for (int i = 0; i < 2; ++i) {
        L.a.codes[i] = cache->codes[i];
        L.a.tok[i] = reinterpret_cast<const __half*>(cache->tok[i]);
        L.a.chan[i] = reinterpret_cast<const __half*>(cache->chan[i]);
        L.a.off[i] = reinterpret_cast<const __half*>(cache->off[i]);
        L.a.resid[i] = reinterpret_cast<const __half*>(cache->resid[i]);
    }
    L.a.q = reinterpret_cast<const __half*>(q);
    L.a.out = out;
    L.a.part = static_cast<float*>(ws);
    L.a.signs = cfg->signs;
    L.a.H = cache->kv_heads;
    L.a.G = G;
    L.a.cap = cache->capacity;
    L.a.nbq = (int)(cache->len / kT);
    L.a.rlen = (int)(cache->len % kT);
    L.a.nsplit = decode_splits(cache);
    const int nbq1 = L.a.nbq > 0 ? L.a.nbq : 1;
    L.a.bps = (nbq1 + L.a.nsplit - 1) / L.a.nsplit;
    L.a.scale = scale > 0.0f ? scale : rsqd_of(cfg->head_dim);
    L.a.rsqd = rsqd_of(cfg->head_dim);
    L.a.sqd = sqd_of(cfg->head_dim);
    L.bh = cache->batch * cache->kv_heads;
    L.st = static_cast<cudaStream_t>(stream);
    return dispatch(cfg->head_dim, cfg->bits, mi, L);
}

size_t kvq_select_signs_workspace_bytes(int32_t n_cand, int64_t n_blocks) {
    if (n_cand < 1 || n_cand > KVQ_SELECT_MAX_CANDIDATES || n_blocks < 1 || n_blocks > INT32_MAX) return 0;
    return (size_t)n_cand * (size_t)n_blocks * sizeof(double);
}

kvq_status kvq_select_signs(const kvq_config* cfg, const uint16_t* x, int64_t n_blocks, const int8_t* signs,
                            int32_t n_cand, double* err, int32_t* best, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("kvq_select_signs");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if (!mi.had || mi.mode == kNaive) return KVQ_ERR_UNSUPPORTED;
    if (!ok_ptr(x) || !ok_ptr(signs) || !ok_ptr(err) || !ok_ptr(best)) return KVQ_ERR_INVALID_ARG;
    if (n_cand < 1 || n_cand > KVQ_SELECT_MAX_CANDIDATES || n_blocks < 1 || n_blocks > INT32_MAX)
        return KVQ_ERR_INVALID_ARG;
    const size_t need = kvq_select_signs_workspace_bytes(n_cand, n_blocks);
    if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return KVQ_ERR_WORKSPACE;
    SelectLaunch L;
    L.a.x = reinterpret_cast<const __half*>(x);
    L.a.signs = signs;
    L.a.part = static_cast<double*>(ws);
    L.a.n_blocks = (int)n_blocks;
    L.a.rsqd = rsqd_of(cfg->head_dim);
    L.a.sqd = sqd_of(cfg->head_dim);
    L.n_cand = n_cand;
    L.err = err;
    L.best = best;
    L.st = static_cast<cudaStream_t>(stream);
    return dispatch(cfg->head_dim, cfg->bits, mi, L);
}

kvq_status kvq_dequantize(const kvq_config* cfg, const kvq_cache* cache, int32_t tensor, int64_t t0, int64_t ntok,
                          float* out, void* stream) {
    NvtxRange nvtx_range("kvq_dequantize");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if ((s = check_cache(cfg, mi, cache)) != KVQ_OK) return s;
    if (tensor != 0 && tensor != 1) return KVQ_ERR_INVALID_ARG;
    if (!ok_ptr(out)) return KVQ_ERR_INVALID_ARG;
    if (t0 < 0 || ntok <= 0 || t0 % kT != 0 || ntok % kT != 0) return KVQ_ERR_INVALID_ARG;
    if (t0 + ntok > (cache->len / kT) * kT) return KVQ_ERR_INVALID_ARG;
    DequantLaunch L;
    L.a.codes = cache->codes[tensor];
    L.a.pairv = tensor;  // V rows of head dim 128 are pair-interleaved
    L.a.tok = reinterpret_cast<const __half*>(cache->tok[tensor]);
    L.a.chan = reinterpret_cast<const __half*>(cache->chan[tensor]);
    L.a.off = reinterpret_cast<const __half*>(cache->off[tensor]);
    L.a.signs = cfg->signs;
    L.a.out = out;
    L.a.cap = cache->capacity;
    L.a.ntok = (int)ntok;
    L.a.blk0 = (int)(t0 / kT);
    L.a.rsqd = rsqd_of(cfg->head_dim);
    L.a.sqd = sqd_of(cfg->head_dim);
    L.bh = cache->batch * cache->kv_heads;
    L.nblk = (int)(ntok / kT);
    L.st = static_cast<cudaStream_t>(stream);
    return dispatch(cfg->head_dim, cfg->bits, mi, L);
}

}  // extern "C"

namespace kvq {
namespace {

// Scratch of kvq_decode_attention_noalloc: a file-scope device array, so the
// entry point needs neither an allocation nor a caller workspace.  Host code
// must not pass `g_noalloc_scratch` itself to a kernel: on the host that name
// is only a stand-in; the device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  Returns nullptr if the lookup fails.
void* noalloc_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace kvq

extern "C" {

kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache* cache, const uint16_t* q,
                                        int32_t q_heads, float scale, float* out, void* stream) {
    NvtxRange nvtx_range("kvq_decode_attention_noalloc");
    ModeInfo mi;
    kvq_status s = check_cfg(cfg, &mi);
    if (s != KVQ_OK) return s;
    if ((s = check_cache(cfg, mi, cache)) != KVQ_OK) return s;
    if (!ok_ptr(q) || !ok_ptr(out)) return KVQ_ERR_INVALID_ARG;
    if (q_heads < cache->kv_heads || q_heads % cache->kv_heads != 0) return KVQ_ERR_INVALID_ARG;
    if (q_heads / cache->kv_heads > kGMax) return KVQ_ERR_UNSUPPORTED;
    // sizes are checked before any CUDA call
    const size_t need = kvq_decode_workspace_bytes(cfg, cache, q_heads);
    if (need == 0 || need > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
    void* ws = noalloc_scratch_ptr();
    if (ws == nullptr) return KVQ_ERR_CUDA;
    // The split kernel writes every partial it later reads, so no part of the
    // shared scratch has to start at zero.
    return kvq_decode_attention(cfg, cache, q, q_heads, scale, out, ws, (size_t)KVQ_NOALLOC_SCRATCH_BYTES, stream);
}

kvq_status kvq_read_device_errors(uint32_t* host_out, int32_t clear) {
    if (host_out == nullptr) return KVQ_ERR_INVALID_ARG;
    if (cudaMemcpyFromSymbol(host_out, g_error_word, sizeof(uint32_t)) != cudaSuccess) return KVQ_ERR_CUDA;
    if (clear) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t)) != cudaSuccess) return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
}

#ifdef KVQ_WAIT_TEST
// Test build only (not declared in kvq.h): scale of the kernels' main-loop
// wait limits; 0 makes every such wait give up at once.
kvq_status kvq_test_set_wait_scale(uint32_t scale) {
    return cudaMemcpyToSymbol(g_wait_scale, &scale, sizeof(scale)) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}
#endif

const char* kvq_status_string(kvq_status status) {
    switch (status) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument";
        case KVQ_ERR_UNSUPPORTED: return "unsupported head_dim, bits or flag set";
        case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
        case KVQ_ERR_WORKSPACE: return "decode workspace missing or too small";
        case KVQ_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

}  // extern "C"
