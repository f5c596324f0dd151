/*
 * kvq.h -- C ABI of libkvq: low-bit KV-cache quantization (norm separation +
 * per-channel block scales, optional randomized Hadamard rotation, optional
 * Normalize-Shift-Normalize) and decode attention over the packed cache,
 * for NVIDIA B200 (sm_100a).
 *
 * Sources the calls follow (page title, section):
 *  - "KV cache INT4 quantization ... nsep+pchan" post, section "Fix
 *    (nsep+pchan)": each K/V vector becomes an FP16 norm plus a unit
 *    direction; the direction is quantized with per-channel scales and
 *    symmetric round-to-nearest codes (+-7 at INT4); a drop-in step in front
 *    of the cache, with no training or calibration.
 *  - "Rotated Runtime Smooth" analysis, master equation and symbol list: the
 *    rotation R = (1/sqrt(K)) [+-1] with R R^T = I, the runtime per-channel
 *    scale s_j = max over tokens of |channel j|, alpha = max|X|/(2^(N-1)-1).
 *  - "NSNQuant" explainer, "Method" (Normalize-Shift-Normalize with side
 *    products s1, o, s2; Hadamard transform) and "Implementation details"
 *    (quantized part plus a full-precision residual that is flushed into the
 *    quantized part when full; attention computed directly from the codes with
 *    the side products folded into the kernel).
 *  - "Activation-guided compensation and orthogonal residuals" abstract:
 *    randomized Hadamard rotation with random sign patterns.
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers unless a comment says "host".
 *    The library never allocates or frees memory; the caller owns every
 *    buffer.  Device pointers must be 16-byte aligned.
 *  - fp16 data is passed as uint16_t bit patterns (IEEE binary16).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    only enqueue work and never synchronize.
 *  - Every argument is checked on the host before anything is enqueued; a
 *    failed check returns an error and changes no state.  Errors reported by
 *    the CUDA runtime at launch are returned as KVQ_ERR_CUDA.
 *  - The library's global state is small and per device: a sticky device
 *    error word (kvq_read_device_errors), per-device flags recording which
 *    kernel attributes have been set, and the fixed scratch array of
 *    kvq_decode_attention_noalloc.  Calls on distinct caches may be made from
 *    several host threads; kvq_decode_attention_noalloc calls that overlap on
 *    the GPU race on the shared scratch (see there).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad size or range */
    KVQ_ERR_UNSUPPORTED = 2, /* head_dim / bits / flag set not built for the GPU */
    KVQ_ERR_CAPACITY = 3,    /* write past the cache capacity */
    KVQ_ERR_WORKSPACE = 4,   /* decode workspace missing or too small */
    KVQ_ERR_CUDA = 5         /* the CUDA runtime reported an error */
} kvq_status;

/* Quantizer flags. */
enum {
    KVQ_NORM_SEP = 1u,    /* split off the FP16 L2 norm; quantize the unit direction */
    KVQ_PER_CHANNEL = 2u, /* per-channel scale over each 128-token block (else per token) */
    KVQ_NSN = 4u,         /* Normalize-Shift-Normalize before quantization */
    KVQ_HADAMARD = 8u,    /* (randomized) Hadamard rotation of the direction */
    KVQ_DQ = 16u          /* NSN only: double quantization of the side parameters o, s1 */
};

#define KVQ_BLOCK_TOKENS 128

/*
 * Quantizer configuration.  Flag sets built for the GPU:
 *   NORM_SEP | PER_CHANNEL            nsep+pchan
 *   NORM_SEP | PER_CHANNEL | HADAMARD randomized Hadamard, then nsep+pchan
 *   0                                  naive per-token absmax
 *   NSN | PER_CHANNEL [| HADAMARD]     NSN (+ Hadamard), per-channel codes
 *   NSN | PER_CHANNEL [| HADAMARD] | DQ   the same with double quantization
 * head_dim in {64, 128}; bits in {2, 3, 4}.
 * DQ (NSNQuant explainer, "Double Quantization (DQ)": the NSN parameters o
 * and s1 are themselves quantized to 4 bits): per 128-token block the means
 * o get symmetric 4-bit codes with one fp16 scale sigma_o = fp16(max|o|/7),
 * and the token scales s1 unsigned 4-bit codes over [lo, lo + 15 step] with
 * lo = fp16(min s1), step = fp16((max s1 - lo) / 15); the encoder subtracts
 * the rebuilt means.  Both go to a block record in off[] (layout below).
 */
typedef struct {
    int32_t head_dim;
    int32_t bits;
    uint32_t flags;
    int32_t reserved;    /* must be 0 */
    const int8_t* signs; /* device [head_dim] of +-1 used by HADAMARD (the same
                            vector rotates K, V, queries and outputs); NULL means
                            all +1, i.e. the plain Hadamard transform */
} kvq_config;

/*
 * The packed cache.  Caller-allocated; index [2] selects K (0) or V (1).
 * Shapes (row-major, B = batch, H = kv_heads, S = capacity, nb = S / 128):
 *   codes[i] uint8  [B][H][S][row_bytes]   row_bytes = kvq_row_bytes(head_dim, bits)
 *   tok[i]   fp16   [B][H][S][ntok]        ntok = kvq_tok_params(flags):
 *                                          nsep: norm; naive: scale; NSN: s1, s2;
 *                                          NSN with DQ: s2
 *   chan[i]  fp16   [B][H][nb][head_dim]   per-channel block scale (PER_CHANNEL, else NULL)
 *   off[i]   fp16   [B][H][nb][kvq_off_words(flags, head_dim)]   (NSN, else NULL):
 *            the per-channel block means, or under DQ the block record:
 *            bytes [0, head_dim/2) the codes of o (e = q + 8, channel 2j in
 *            the low nibble of byte j), [head_dim/2, head_dim/2 + 64) the
 *            codes of s1 (q in 0..15, token 2j in the low nibble of byte j),
 *            then fp16 sigma_o, lo, step, zeros up to a multiple of 16 bytes;
 *            o_hat = (e - 8) sigma_o, s1_hat = lo + q step
 *   resid[i] fp16   [B][H][128][head_dim]  residual tokens not yet quantized
 * Code layout per token row: offset-binary e = q + 2^(bits-1) (never 0);
 *   INT4 byte j = e[2j] | e[2j+1] << 4; INT2 byte j = e[4j] | e[4j+1] << 2 |
 *   e[4j+2] << 4 | e[4j+3] << 6; INT3 = head_dim/4 bytes of (e & 3) in the
 *   INT2 layout followed by head_dim/8 bytes whose bit i of byte j is bit 2
 *   of e[8j+i].
 * V codes of head_dim 128 are stored pair-interleaved (the layout the decode
 *   kernel's value operand takes): the rows of tokens 2k and 2k+1 form a
 *   pair block of 2*row_bytes bytes at the place of those two rows, whose
 *   little-endian 32-bit word u holds bytes 2u, 2u+1 of row 2k in its low
 *   half and of row 2k+1 in its high half; at INT4 the 16-byte chunk c of
 *   pair block k is stored at chunk c ^ (2*(k & 1)).  K codes, and V codes
 *   of head_dim 64, are plain token rows.
 * `len` is the number of tokens stored: tokens [0, 128*floor(len/128)) are in
 * the quantized blocks, the remaining len % 128 are residual slots
 * 0 .. len%128-1.  The library updates `len` on the host struct after a
 * successful enqueue of kvq_quantize_block or kvq_append_token.
 */
typedef struct {
    int32_t batch, kv_heads, head_dim, capacity;
    int64_t len;
    uint8_t* codes[2];
    uint16_t* tok[2];
    uint16_t* chan[2];
    uint16_t* off[2];
    uint16_t* resid[2];
} kvq_cache;

/* Bytes of one packed token row; 0 for an unsupported (head_dim, bits). */
int32_t kvq_row_bytes(int32_t head_dim, int32_t bits);

/* fp16 per-token parameters stored for a flag set (ntok above); -1 if the
   flag set is not built for the GPU. */
int32_t kvq_tok_params(uint32_t flags);

/* fp16 words per block of the off[] arrays for a flag set and head_dim: the
   head_dim means, or under DQ the record's bytes / 2; 0 without NSN; -1 if
   the flag set or head_dim is not built for the GPU. */
int32_t kvq_off_words(uint32_t flags, int32_t head_dim);

/*
 * Random signs of the randomized Hadamard rotation ("random sign patterns",
 * randomized Hadamard abstract; R = (1/sqrt(K))[+-1], Rotated Runtime Smooth
 * symbol list).  HOST function: writes head_dim values of +-1 to host_out.
 * sign_c = -1 iff bit 63 of the c-th SplitMix64 output from state `seed` is
 * set (SplitMix64: Steele, Lea & Flood 2014).  Copy the result to the device
 * for kvq_config.signs.  KVQ_ERR_INVALID_ARG if host_out is NULL or
 * head_dim < 1.
 */
kvq_status kvq_make_signs(uint64_t seed, int32_t head_dim, int8_t* host_out);

/*
 * Quantize ntok tokens of K and of V into the cache blocks starting at token
 * t0 (the prefill / bulk path).  nsep+pchan post "Fix (nsep+pchan)" (norm +
 * direction, per-channel scales, codes +-qmax); NSNQuant "Method" (NSN,
 * Hadamard); Rotated Runtime Smooth symbol list (per-channel absmax over
 * tokens, qmax = 2^(N-1)-1).
 *   k, v   fp16 [B][H][ntok][head_dim], contiguous
 *   t0     multiple of 128; ntok > 0 and a multiple of 128
 * A persistent grid (a few CTAs per SM) takes the (b, h, block, tensor)
 * tiles in turn; each tile of 128 x head_dim fp16 values is read from HBM
 * once and its codes, per-token parameters and per-block channel
 * scales/means are written once.
 * On success len = max(len, t0 + ntok).
 * Errors: INVALID_ARG (null/misaligned pointers, t0 or ntok not multiples of
 * 128, or a range that overlaps residual tokens that are still held, i.e.
 * t0 + ntok > 128*floor(len/128) while len % 128 != 0); CAPACITY
 * (t0 + ntok > capacity); UNSUPPORTED; CUDA.
 */
kvq_status kvq_quantize_block(const kvq_config* cfg, kvq_cache* cache,
                              const uint16_t* k, const uint16_t* v,
                              int64_t t0, int64_t ntok, void* stream);

/*
 * Append one token per (b, h) to the residual (NSNQuant "Implementation
 * details": full-precision residual flushed into the quantized part when
 * full).  k_new, v_new fp16 [B][H][head_dim].  The token goes to residual
 * slot len % 128; when that slot is 127 the call instead quantizes the 128
 * residual tokens into block floor(len/128) exactly as kvq_quantize_block
 * would, which empties the residual.  On success len += 1.
 * Errors: INVALID_ARG; CAPACITY (len + 1 > capacity); UNSUPPORTED; CUDA.
 */
kvq_status kvq_append_token(const kvq_config* cfg, kvq_cache* cache,
                            const uint16_t* k_new, const uint16_t* v_new, void* stream);

/* Workspace bytes kvq_decode_attention needs for this cache and q_heads
   (partial softmax states of the sequence splits); 0 on invalid arguments.
   At head dim 128 the size depends on the current device's SM count (the
   persistent grid is at most 4 CTAs per SM): size it on the device the
   decode runs on.  Each call writes every partial state it reads, so the
   workspace needs no initialization. */
size_t kvq_decode_workspace_bytes(const kvq_config* cfg, const kvq_cache* cache, int32_t q_heads);

/*
 * Decode attention of one query token per sequence over the cache:
 *   out[b, j] = sum_{t < len} softmax_t(scale * q[b, j] . x_hat^K_t) x_hat^V_t
 * with query head j reading kv head j / (q_heads / kv_heads).  Quantized
 * tokens are read as packed codes plus their side parameters and are never
 * expanded in memory (NSNQuant "Implementation details": the side products
 * are folded into the attention kernel); residual tokens are attended at
 * their fp16 values.  x_hat is the tensor kvq_dequantize rebuilds.
 *   q     fp16 [B][q_heads][head_dim]; q_heads a multiple of kv_heads,
 *         q_heads / kv_heads <= 8
 *   scale softmax scale; <= 0 selects 1/sqrt(head_dim)
 *   out   fp32 [B][q_heads][head_dim]; len == 0 gives zeros
 *   ws    workspace of at least kvq_decode_workspace_bytes() (contents
 *         need no initialization); calls that share a workspace must not
 *         overlap in time
 * Stream order: at head dim 128 the call's kernels are launched as
 * programmatic dependents (their launch overlaps the tail of the kernel
 * ahead of them in the stream; they wait for it to finish before reading
 * or writing any memory), so ordinary stream order holds for the caller.
 * Errors: INVALID_ARG; WORKSPACE; UNSUPPORTED; CUDA.
 */
kvq_status kvq_decode_attention(const kvq_config* cfg, const kvq_cache* cache,
                                const uint16_t* q, int32_t q_heads, float scale,
                                float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Rebuild fp32 values of quantized tokens [t0, t0 + ntok) of K (tensor 0) or
 * V (tensor 1): out fp32 [B][H][ntok][head_dim].  x_hat = norm * (q * sigma)
 * (nsep); inverse rotation for HADAMARD; s1 * (s2 * sqrt(d) R^T (q * sigma) +
 * o) for NSN (NSNQuant "Method": the side products rebuild the tensor).
 * Errors: INVALID_ARG (t0, ntok not multiples of 128, or the range is not
 * inside the quantized part); UNSUPPORTED; CUDA.
 */
kvq_status kvq_dequantize(const kvq_config* cfg, const kvq_cache* cache, int32_t tensor,
                          int64_t t0, int64_t ntok, float* out, void* stream);

/*
 * Sign-pattern selection for the randomized Hadamard rotation
 * ("Activation-guided compensation and orthogonal residuals" abstract:
 * sampling several random sign patterns improves the choice of the
 * transform; random signs keep persistent outlier channels from adding up).
 * Quantizes a sample with each candidate sign vector exactly as
 * kvq_quantize_block does (cfg.signs is ignored), rebuilds it as
 * kvq_dequantize does, and measures the reconstruction error
 *   err[k] = sum over the sample's blocks, in order, of the pairwise sum
 *            over the block's tokens of the pairwise sum over channels of
 *            (x_hat - x)^2, in fp64;
 * best = the index of the smallest err (the lowest index among equal ones).
 *   cfg     flags with KVQ_HADAMARD (nsep+pchan or NSN); head_dim, bits as usual
 *   x       fp16 [n_blocks][128][head_dim], the sample (for instance the
 *           first block of every (batch, kv head) slice of a prefill)
 *   signs   int8 [n_cand][head_dim] of +-1 (e.g. kvq_make_signs of n_cand
 *           seeds, copied to the device), 1 <= n_cand <= KVQ_SELECT_MAX_CANDIDATES
 *   err     fp64 [n_cand] out;  best  int32 [1] out
 *   ws      workspace of kvq_select_signs_workspace_bytes(n_cand, n_blocks)
 *           bytes (the per-block errors; needs no initialization)
 * Errors: INVALID_ARG; UNSUPPORTED (no HADAMARD flag, or the naive mode);
 * WORKSPACE; CUDA.
 */
#define KVQ_SELECT_MAX_CANDIDATES 256
size_t kvq_select_signs_workspace_bytes(int32_t n_cand, int64_t n_blocks);
kvq_status kvq_select_signs(const kvq_config* cfg, const uint16_t* x, int64_t n_blocks, const int8_t* signs,
                            int32_t n_cand, double* err, int32_t* best, void* ws, size_t ws_bytes, void* stream);

/*
 * Decode attention that allocates nothing and needs no caller workspace.
 * The pages have no counterpart to this call; it exists for callers that are
 * handed only their input and output buffers and cannot allocate device
 * memory: an operator plugin inside an inference engine that plans all
 * device memory ahead of time, or code on a latency-critical path where
 * cudaMalloc would synchronize the device.
 * Same arguments, results and errors as kvq_decode_attention, minus the
 * workspace.  The split-K partial results go to a scratch array of
 * KVQ_NOALLOC_SCRATCH_BYTES (32 MiB) that the library holds in device memory
 * on every GPU that loads it, until the process exits.  A call whose
 * workspace need (kvq_decode_workspace_bytes) exceeds that size returns
 * KVQ_ERR_WORKSPACE before enqueuing anything.
 * The first call on a device looks up the array's device address on that
 * device (it must be the current device); make that first call before any
 * stream capture.  All calls on a device share the one array, which keeps the
 * last call's contents: calls that overlap in time on the GPU (different
 * streams, or different host threads) race and corrupt each other's results.
 * The call never runs cudaMalloc, cudaFree or any allocating routine.
 */
#define KVQ_NOALLOC_SCRATCH_BYTES (32u << 20)
kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache* cache,
                                        const uint16_t* q, int32_t q_heads, float scale,
                                        float* out, void* stream);

/*
 * Read (and, if clear != 0, reset) the sticky device error word of the
 * current device: bit 0 = a kernel gave up waiting for a TMA tile, bit 1 = a
 * kernel gave up waiting on a barrier.  Kernels that give up leave the
 * results of that call undefined.  HOST call; synchronizes the device.
 * Errors: INVALID_ARG (host_out NULL); CUDA.
 */
kvq_status kvq_read_device_errors(uint32_t* host_out, int32_t clear);

/* Static description of a status code. */
const char* kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
