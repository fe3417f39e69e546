/*
 * kvq.h - C ABI of libkvq: RoPE-aware packed KV-cache quantization and
 * packed-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ),
 * abstract. Per (layer, KV head): a label-free energy score of each RoPE 2-D
 * block, greedy integer bit widths by marginal gain under a matched K/V bit
 * budget (KxVy), quantization built on TurboQuant-MSE (TQ-MSE), and a
 * packed-cache serving path whose decode attention reads the packed cache.
 * The abstract leaves the energy formula, the distortion model, the
 * codebooks, the norm and the packing open; the readings adopted are stated
 * at each entry point below.
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller allocates and frees every buffer (caches, plans,
 *     workspace, lengths, status word). The library never allocates device
 *     memory and keeps no pointer after a call returns.
 *   - Pointers named *_dev are device pointers; *_host are host pointers.
 *     "Device array of pointers" means a device buffer holding device
 *     addresses (64-bit each).
 *   - Asynchrony: calls enqueue work on `stream` and return once it is
 *     launched. kvq_alloc_bits is the exception: it synchronizes `stream`
 *     once (it needs the energies on the host).
 *   - Errors: a negative return means nothing was launched;
 *     kvq_last_error() gives a message (thread-local). Problems that only
 *     the device can see set bits of *status_dev with an atomic OR
 *     (KVQ_FLAG_*); kernels never trap and never wait without a bound.
 *   - Supported shapes: head_dim = 128; bits_k and bits_v in 1..8; b_max = 8;
 *     n_q_heads a multiple of n_kv_heads with G = n_q_heads / n_kv_heads <= 16.
 *   - Thread safety: calls on different streams may run concurrently; the
 *     library's mutable global state is kvq_last_error(), the two
 *     process-wide decode modes (kvq_set_decode_deterministic,
 *     kvq_debug_decode_stall) and the fixed scratch of
 *     kvq_decode_attn_noalloc (whose calls must not overlap).
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

/* A cudaStream_t (the runtime's stream handle type). 0 = legacy stream. */
typedef struct CUstream_st* kvq_stream_t;

/* Return codes. */
#define KVQ_OK 0
#define KVQ_ERR_ARG (-1)          /* bad argument (null pointer, range, size) */
#define KVQ_ERR_UNSUPPORTED (-2)  /* valid but unsupported shape (head_dim != 128) */
#define KVQ_ERR_WORKSPACE (-3)    /* workspace smaller than required */
#define KVQ_ERR_CUDA (-4)         /* a CUDA runtime call failed */

/* Device status flags, OR-ed into *status_dev (a uint32 the caller zeroes). */
#define KVQ_FLAG_CAPACITY 1u   /* append past cap_tokens (sequence skipped), or len > max_len */
#define KVQ_FLAG_NONFINITE 2u  /* a token had a NaN/Inf coordinate: stored as norm 0, codes 0 */
#define KVQ_FLAG_NORM_SAT 4u   /* a norm overflowed fp16: stored as 65504 */
#define KVQ_FLAG_TIMEOUT 8u    /* a bounded wait ran out: output invalid */
#define KVQ_FLAG_BAD_PLAN 16u  /* a plan record failed its device check (magic, shape, or an
                                  order / segment / schedule that does not follow from
                                  its widths): kvq_quantize_append stores no token with
                                  it, a fused append (kvq_append_decode) may store
                                  undefined codes in the token's tile record, the length
                                  still advances, and decode output is invalid */
#define KVQ_FLAG_BAD_PAGE 32u  /* paged cache: a tile past the block table or a page id outside
                                  the pool (appends skip it; decode output is invalid) */

/* Input element types. */
#define KVQ_BF16 0
#define KVQ_FP16 1
#define KVQ_FP32 2

/* kvq_append_decode step flags. */
#define KVQ_STEP_EARLY 1u  /* see kvq_append_decode */
#define KVQ_STEP_ROPE 2u   /* see kvq_append_decode */

/* Allocation modes. */
#define KVQ_ALLOC_GREEDY 0   /* Block-GTQ: greedy marginal-gain widths per RoPE block */
#define KVQ_ALLOC_UNIFORM 1  /* every block gets bits_k (same bytes; comparator) */
#define KVQ_ALLOC_ROTATE_KEYS 0x100 /* OR-ed into alloc_mode: rotate keys inside each group of
                                       blocks of one width before coding (plan field k_rot) */

typedef struct {
  int32_t head_dim;    /* must be 128 */
  int32_t n_kv_heads;  /* KV heads per layer, >= 1 */
  int32_t bits_k;      /* key budget, bits per dimension, 1..8 (K in KxVy) */
  int32_t bits_v;      /* value width, bits per dimension, 1..8 (V in KxVy) */
  int32_t b_max;       /* largest width of one block, must be 8 */
  int32_t alloc_mode;  /* KVQ_ALLOC_GREEDY or KVQ_ALLOC_UNIFORM, optionally | KVQ_ALLOC_ROTATE_KEYS */
  uint64_t v_seed;     /* seed of the value sign flips */
} kvq_cfg;

/*
 * Plan record: one per (layer, KV head), KVQ_PLAN_BYTES bytes, plain data
 * (copy it with memcpy; it holds no pointer). Little-endian layout:
 *   off   0  uint32  magic = KVQ_PLAN_MAGIC
 *   off   4  int32   bits_k
 *   off   8  int32   bits_v
 *   off  12  int32   n_ranks        stored (nonzero-width) blocks
 *   off  16  int32   layer
 *   off  20  int32   kv_head
 *   off  24  int32   words_k        K code words per 32-token tile = 128 * bits_k
 *   off  28  int32   words_v        V code words per 32-token tile = 128 * bits_v
 *   off  32  float   g[64]          quantize scale of block j: fp32(1/a_j), 0 if a_j = 0
 *   off 288  float   a_hat[64]      dequantize scale of block j: fp32(a_j)
 *   off 544  uint8   width[64]      bits of block j (0..8)
 *   off 608  uint8   order[64]      plan rank -> block index (ranks >= n_ranks unused)
 *   off 672  uint16  seg_off[65]    rank -> first word of its K segment in a tile record
 *   off 802  uint8   n_half         decode schedule: groups of <= 4 equal-width ranks
 *   off 803  uint8   pad
 *   off 804  uint8   hs_width[32]
 *   off 836  uint8   hs_rank0[32]
 *   off 868  uint8   hs_count[32]
 *   off 900  uint32  v_sign[4]      bit i set <=> value sign s_i = -1
 *   off 916  uint32  pad
 *   off 920  double  energy_sum     sum of the 64 block energies, fp64 in block order
 *   off 928  uint8   n_class        decode schedule: runs of half steps of one width
 *   off 936  uint8   cls_w[8]
 *   off 944  uint8   cls_hs0[8]     first half step of the class
 *   off 952  uint8   cls_nhs[8]     half steps in the class
 *   off 960  uint8   cls_last[8]    blocks in the class's last half step
 *   off 968  uint16  cls_seg0[8]    first K word of the class in a tile record
 *   off 984  uint32  k_sign[4]      key rotation: bit P set <=> sign of plan position P is -1
 *   off 1000 uint8   k_rot          1: keys rotated inside each width group (see below)
 *   off 1001 .. 1023 zero
 *
 * Key rotation (KVQ_ALLOC_ROTATE_KEYS; the alternative reading of "built on
 * TQ-MSE" for keys, which spreads outlier coordinates before coding). Plan
 * position P = 2 r + e is coordinate order[r] + 64 e. A width group (the
 * ranks of one class) holds 2 n positions, cut into chunks by the binary
 * expansion of 2 n (largest first). Per token, after z_i = (k_i * r) * g_j
 * as without rotation: u_P = s_P z_P, the fp32 FWHT graph over each chunk
 * (stages h = 1, 2, ... < size, pairs (P, P + h) with (P - chunk start) & h
 * == 0 become (a + b, a - b)), y_P = fp32(h_P * c(size)), c(2^e) =
 * 2^-floor(e/2) times fp32(sqrt(1/2)) for odd e; y_P is coded at the group's
 * width into the slot of coordinate order[r] + 64 e. Signs: s_P = -1 iff bit
 * 63 of SplitMix64(key, 128 + P) is set (key as for the value signs).
 * Decode rotates the query the same way (q~ = c H (s . q') per chunk), so
 * q . k_hat needs no inverse transform per token.
 */
#define KVQ_PLAN_BYTES 1024
#define KVQ_PLAN_MAGIC 0x5051564Bu /* "KVQP" */

/* Library version string. */
KVQ_API const char* kvq_version(void);

/* Message of the last negative return on the calling thread ("" if none). */
KVQ_API const char* kvq_last_error(void);

/* Size of one plan record (KVQ_PLAN_BYTES). */
KVQ_API size_t kvq_plan_bytes(void);

/*
 * Bytes of one 32-token tile record for the budget of `cfg`:
 * 512 * (bits_k + bits_v) + 128. Layout (little-endian 32-bit words):
 *   [K: 128 bits_k words][V: 128 bits_v words][K norms: 32 fp16][V norms: 32 fp16]
 * K part: one segment of 2w words per stored block, in plan order
 * (order[], seg_off[]); segment words hold 32 fields of 2w bits, token
 * position t of the tile at bit (4 (t mod 8) + t div 8) * 2w, low w bits the
 * code of coordinate j, high w bits the code of j + 64.
 * V part: 128 segments of bits_v words (rotated coordinate p at word
 * 128 bits_k + p bits_v), token position t at bit
 * (8 ((t mod 8) div 2) + 2 (t div 8) + (t mod 2)) * bits_v.
 * Code bits of positions holding no token are zero.
 * This is the reading adopted for the pages' "packed K3V3" cache: exactly
 * b_K + b_V bits per dimension plus two fp16 norms per token and head
 * (K3V3: 100 bytes per token and KV head).
 */
KVQ_API size_t kvq_tile_bytes(const kvq_cfg* cfg);

/*
 * Bytes of the packed cache of one (sequence, layer) holding up to
 * cap_tokens tokens: ceil(cap_tokens / 32) * n_kv_heads * kvq_tile_bytes.
 * Tile tau (tokens 32 tau .. 32 tau + 31) of KV head h is the record at byte
 * offset (tau * n_kv_heads + h) * tile_bytes. Returns 0 for an invalid cfg.
 * The base address must be 16-byte aligned (kernels flag BAD_PLAN and skip
 * a sequence whose cache is not).
 */
KVQ_API size_t kvq_cache_bytes(const kvq_cfg* cfg, int64_t cap_tokens);

/* Workspace bytes kvq_alloc_bits needs: n_kv_heads * 64 * 16 (+ alignment). */
KVQ_API size_t kvq_alloc_workspace_bytes(const kvq_cfg* cfg);

/*
 * Workspace bytes kvq_decode_attn needs for `batch` sequences on the current
 * device: a region of split-K records (m, l, o[128]) bounded by one record
 * set per CTA slot of the device (or per sequence x KV head, if there are
 * more) for up to 16 query heads, then, at fixed distances from the end of
 * the workspace, one block per (sequence, KV head) of arrival counters and
 * 16 exponent buckets per query head (135,296 bytes). The size depends on
 * batch x n_kv_heads only, not on max_len or n_q_heads (kept as arguments).
 * Without a usable device it returns an upper bound.
 * Returns 0 for invalid arguments.
 */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cfg* cfg, int batch, int n_q_heads,
                                  int64_t max_len);

/*
 * Block energies and bit allocation for one layer: Block-GTQ's label-free
 * per-RoPE-block energy score and greedy marginal-gain integer widths
 * ("RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract).
 * Readings adopted:
 *   energy   E_j = (1/T) sum_t (k_{t,j}^2 + k_{t,j+64}^2) over the T given
 *            keys, each square taken on a 2^-32 fixed-point grid
 *            (floor(k^2 2^32), saturating at 2^64-1) and summed exactly as an
 *            integer, so the result does not depend on summation order;
 *   D(b)     Lloyd-Max MSE of a unit Gaussian with 2^b levels, D(0) = 1;
 *   greedy   64 bits_k steps from all-zero widths; each adds 1 bit to the
 *            block of largest E_j (D(b_j) - D(b_j + 1)) below b_max; ties to
 *            the lowest index;
 *   scales   a_j = sqrt(E_j / (2 sum_l E_l)); g_j = fp32(1/a_j), a_hat_j = fp32(a_j);
 *   signs    value sign s_i = -1 iff bit 63 of SplitMix64(key, i) is set,
 *            key = SplitMix64(v_seed, layer * 2^32 + kv_head) (n-th output of
 *            the stream seeded with s: mix(s + (n + 1) 0x9E3779B97F4A7C15)).
 * k_dev: keys [n_tokens][n_kv_heads][128] of type k_dtype (post-RoPE; the
 *        energy is RoPE-invariant). n_tokens >= 1.
 * ws_dev: >= kvq_alloc_workspace_bytes(cfg) bytes (contents overwritten).
 * plans_dev: out, n_kv_heads plan records (contiguous).
 * plans_host: optional out (may be NULL), same records on the host.
 * energy_host: optional out (may be NULL), E[n_kv_heads][64] as fp64.
 * status_dev: optional (may be NULL); NONFINITE if a key was not finite
 *        (its square counts 0).
 * Synchronizes `stream` once. Returns KVQ_OK or a negative code.
 */
KVQ_API int kvq_alloc_bits(const kvq_cfg* cfg, int layer, const void* k_dev, int k_dtype,
                   int64_t n_tokens, void* ws_dev, size_t ws_bytes, void* plans_dev,
                   void* plans_host, double* energy_host, uint32_t* status_dev,
                   kvq_stream_t stream);

/*
 * Host-only plan builder from given energies (no GPU work): the greedy,
 * scales and signs of kvq_alloc_bits for E_host[n_heads][64], writing
 * n_heads plan records to plans_host (head h gets kv_head = h).
 */
KVQ_API int kvq_plan_build(const kvq_cfg* cfg, int layer, const double* E_host, int n_heads,
                   void* plans_host);

/*
 * The library's own Gaussian Lloyd-Max tables for `bits` in 1..8 (host, no
 * GPU): 2^bits fp16-exact centroids (as float), 2^bits - 1 fp32 thresholds
 * (midpoints of the centroids), and D(bits). Any output may be NULL.
 */
KVQ_API int kvq_codebook(int bits, float* centroids, float* thresholds, double* distortion);

/*
 * Host check of one plan record before it is uploaded (host memory): magic,
 * bits against cfg, word counts, widths in 0..8 summing to 64 bits_k, finite
 * non-negative scales, k_rot in {0, 1}, and every field that follows from
 * the widths (plan order, segment offsets, half steps, classes) equal to what
 * the widths give. The kernels check only the magic and the shape fields, so
 * a plan that was not built by this library should pass here first.
 * Returns KVQ_OK, or KVQ_ERR_ARG with the first inconsistency in
 * kvq_last_error().
 */
KVQ_API int kvq_plan_check(const kvq_cfg* cfg, const void* plan_host);

/*
 * Query-weighted allocation (a variant; the pages' score is key-only and
 * label-free). The logit q . k is a sum of 2-D RoPE block terms q_j . k_j, so
 * the error of key block j reaches the logit scaled by the query's block
 * energy; weighting the greedy by calibration queries minimises
 * sum_j W_j E_j D(b_j), the expected squared logit error, instead of
 * sum_j E_j D(b_j).
 *
 * kvq_block_energy: the exact block energy E[h][j] (as in kvq_alloc_bits) of
 *   any x_dev [n_tokens][n_heads][128] of type dtype, e.g. calibration
 *   queries; energy_host: out, fp64 [n_heads][64]; ws_dev >=
 *   kvq_energy_workspace_bytes(n_heads) bytes (overwritten); status_dev
 *   optional (NONFINITE). Synchronizes `stream` once.
 * kvq_plan_build_weighted: kvq_plan_build for the n_kv_heads KV heads with
 *   the widths of the greedy on E_j W_j (fp64 products) and the key scales
 *   of E. E_host: key energies [n_kv_heads][64]; Eq_host: query energies
 *   [n_q_heads][64] (kvq_block_energy of calibration queries); W[h] is the
 *   mean over KV head h's query group, (1/G) sum_{g<G} Eq[h G + g] summed
 *   in increasing g, G = n_q_heads / n_kv_heads.
 * Return KVQ_OK or a negative code (size query: 0 if invalid).
 */
KVQ_API size_t kvq_energy_workspace_bytes(int n_heads);
KVQ_API int kvq_block_energy(const void* x_dev, int dtype, int64_t n_tokens, int n_heads,
                             void* ws_dev, size_t ws_bytes, double* energy_host,
                             uint32_t* status_dev, kvq_stream_t stream);
KVQ_API int kvq_plan_build_weighted(const kvq_cfg* cfg, int layer, const double* E_host,
                                    const double* Eq_host, int n_q_heads, void* plans_host);

/*
 * Quantize and append n_new tokens per sequence to the packed cache
 * (Block-GTQ keys on TQ-MSE, uniform TQ-MSE values). Per token and KV head:
 *   keys:   n = fp16(sqrt(sum k_i^2)) (fixed fp32 order), r = 1/n,
 *           z_i = (k_i r) g_j, code_i = #{thresholds of width b_j below z_i};
 *   values: y = H (s . v) (Walsh-Hadamard, fp32 butterflies h = 1..64),
 *           n = fp16 norm of v, z_i = y_i r, codes at width bits_v;
 * all decisions in IEEE fp32 without fused multiply-add, so codes are
 * reproducible bit for bit.
 * plans_dev: device array of `batch` pointers, entry b -> the n_kv_heads
 *        plan records used for sequence b (usually the same layer's plans).
 * k_dev, v_dev: [batch][n_new][n_kv_heads][128] of type `dtype`.
 * cache_dev: device array of `batch` pointers to each sequence's cache
 *        (kvq_cache_bytes(cfg, cap_tokens) bytes, 16-byte aligned).
 * len_dev: int32 [batch]; token positions len..len+n_new-1 are written and
 *        len is then increased by n_new. A sequence with len + n_new >
 *        cap_tokens is skipped (len unchanged) and CAPACITY is flagged.
 * status_dev: required.
 * Tokens already in a tile keep their bits; positions past the new length
 * are zero in a tile that held no tokens and otherwise keep their bits (zero
 * in a cache that was zero-filled and only appended to). Returns KVQ_OK or
 * a negative code.
 */
KVQ_API int kvq_quantize_append(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                        const void* v_dev, int dtype, int batch, int n_new,
                        void* const* cache_dev, int32_t* len_dev, int64_t cap_tokens,
                        uint32_t* status_dev, kvq_stream_t stream);

/*
 * Fused RoPE + quantize-append: k_dev holds pre-RoPE keys;
 * the key of the token at cache position t is first rotated by RoPE at
 * position t with theta_j = rope_base^(-2j/128) (block j = coordinates j,
 * j + 64): angles in fp64, cos and sin rounded once to fp32, the 2-D
 * rotation in fp32 with every product and sum rounded. The rotated key is
 * then quantized exactly as by kvq_quantize_append (the cache holds post-RoPE
 * codes, so decode is unchanged). Same arguments otherwise; rope_base > 1.
 * "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the keys
 * enter the cache after RoPE; the rotation arithmetic is a reading of ours.
 */
KVQ_API int kvq_quantize_append_rope(const kvq_cfg* cfg, const void* const* plans_dev,
                                     const void* k_dev, const void* v_dev, int dtype, int batch,
                                     int n_new, void* const* cache_dev, int32_t* len_dev,
                                     int64_t cap_tokens, double rope_base, uint32_t* status_dev,
                                     kvq_stream_t stream);

/*
 * Decode attention straight from the packed cache: for sequence b and query
 * head h (KV head h / G),
 *   o_h = sum_t softmax_t(q_h . k_hat_t / sqrt(128)) v_hat_t
 * over the len_dev[b] cached tokens, with k_hat and v_hat the dequantized
 * keys and values (k_hat_i = n^K a_hat_j c_{b_j}[code_i];
 * v_hat = n^V (1/128) s . (H c_{bits_v}[codes])). Split-K over the context:
 * each CTA unpacks its tiles in registers, forms the logits of all G query
 * heads of its KV head, keeps an online softmax and accumulates P V in the
 * rotated value domain; each split adds its rescaled sums into exponent
 * buckets in L2 and the last split of a (sequence, KV head) sums the
 * buckets and applies the inverse rotation. One kernel launch; fp32
 * accumulation; the atomic sum order varies, so repeated calls agree to fp32
 * rounding, not bit for bit.
 * plans_dev, cache_dev: as for kvq_quantize_append. The kernel uses
 *        programmatic dependent launch and reads the plans (and their
 *        pointer array) before the previous kernel on the stream has ended,
 *        so that kernel must not write them.
 * len_dev: int32 [batch], each <= max_len (a larger value is clamped to
 *        max_len and flags CAPACITY). A sequence of length 0 gives o = 0.
 * q_dev: [batch][n_q_heads][128] of type q_dtype (post-RoPE queries).
 * out_dev: fp32 [batch][n_q_heads][128].
 * ws_dev: >= kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len)
 *        bytes, 16-byte aligned, zero-filled once before its first use
 *        (KVQ_ERR_ARG if misaligned). Only the per-(sequence, KV head)
 *        blocks at the end of the workspace must be zero when a call starts;
 *        every completed call leaves the blocks it used at zero, and the
 *        split records (written before they are read) never reach into the
 *        blocks of a call with at most as many sequences x KV heads. So one
 *        workspace, sized for the largest batch x n_kv_heads, serves any
 *        sequence of calls on one stream whatever their max_len, query
 *        heads or bit budget; calls that overlap on the GPU must use
 *        different workspaces.
 * status_dev: required.
 * Returns KVQ_OK or a negative code.
 */
KVQ_API int kvq_decode_attn(const kvq_cfg* cfg, const void* const* plans_dev,
                    const void* const* cache_dev, const int32_t* len_dev, int batch,
                    int64_t max_len, const void* q_dev, int q_dtype, int n_q_heads,
                    float* out_dev, void* ws_dev, size_t ws_bytes, uint32_t* status_dev,
                    kvq_stream_t stream);

/*
 * Context-sharded decode (no counterpart in the pages, whose serving path
 * runs on one GPU): a sequence whose cache is split by token ranges over
 * several caches (e.g. one per GPU) is decoded by one kvq_decode_attn_partial
 * per range and one kvq_combine_partials over their records. Softmax over
 * the union of ranges is the log-sum-exp-weighted mix of the per-range
 * results, so the combined output is the kvq_decode_attn output over all
 * tokens (to fp32 rounding). Each range's cache is an ordinary cache
 * holding that range's tokens (post-RoPE keys keep their global positions);
 * len_dev holds the range lengths.
 *
 * kvq_decode_attn_partial: arguments as kvq_decode_attn, but instead of
 *   outputs it writes one record per (sequence, query head) to rec_dev
 *   (fp32 [batch][n_q_heads][132], 16-byte aligned): rec[0] = m,
 *   rec[1] = l, rec[2..3] unused, rec[4..131] = o_rot, meaning
 *   sum_t 2^(s_t - m) = l and sum_t 2^(s_t - m) n^V_t c[vcode_t] = o_rot over
 *   the range's tokens, s_t the base-2 logit q.k_hat_t log2(e) / sqrt(128),
 *   o_rot still in the rotated value domain. An empty range gives
 *   m = -inf, l = 0, o_rot = 0. m is any reference exponent (not
 *   necessarily the range's max); only 2^m (l, o_rot) is defined.
 * kvq_combine_partials: recs_dev = the n_parts record arrays stacked
 *   (fp32 [n_parts][batch][n_q_heads][132], 16-byte aligned, e.g. the result
 *   of an all-gather); plans_dev as for kvq_decode_attn (the value signs);
 *   out_dev fp32 [batch][n_q_heads][128] = s . H o_rot_total / (128 l_total)
 *   after merging the records like split results; 0 where every range was
 *   empty. One launch, no workspace.
 * Both return KVQ_OK or a negative code.
 */
KVQ_API int kvq_decode_attn_partial(const kvq_cfg* cfg, const void* const* plans_dev,
                                    const void* const* cache_dev, const int32_t* len_dev,
                                    int batch, int64_t max_len, const void* q_dev, int q_dtype,
                                    int n_q_heads, float* rec_dev, void* ws_dev, size_t ws_bytes,
                                    uint32_t* status_dev, kvq_stream_t stream);
KVQ_API int kvq_combine_partials(const kvq_cfg* cfg, const void* const* plans_dev, int n_parts,
                                 const float* recs_dev, int batch, int n_q_heads, float* out_dev,
                                 kvq_stream_t stream);

/*
 * Test hook (no counterpart in the paper): with cycles > 0, every later
 * packed decode launch (kvq_decode_attn and the calls built on it) first
 * waits `cycles` clock cycles on a shared-memory barrier that nothing
 * arrives on. The wait runs out, the launch sets KVQ_FLAG_TIMEOUT in
 * *status_dev, lets the tile copies it already issued land, skips its tiles
 * and completes normally (its outputs are then meaningless), which exercises
 * the path every bounded wait of the kernels takes when it gives up. 0
 * restores normal launches. Process-wide; for tests only. Returns KVQ_OK or
 * KVQ_ERR_ARG.
 */
KVQ_API int kvq_debug_decode_stall(long long cycles);

/*
 * Deterministic decode (no counterpart in the paper; for reproducible
 * debugging). on != 0: every later packed decode launch of the process
 * (kvq_decode_attn, kvq_append_decode, the paged and partial forms) merges
 * its split records in split order in the last split, instead of summing the
 * splits in exponent buckets by L2 atomics whose order varies from run to
 * run, so repeated calls on the same inputs give the same bits. It costs a
 * few microseconds per launch (one CTA per sequence and KV head reads every
 * split record). on = 0 restores the default. Returns KVQ_OK.
 */
KVQ_API int kvq_set_decode_deterministic(int on);

/*
 * Recent-token window ("RoPE-Aware Bit Allocation for KV-Cache
 * Quantization", abstract: the paper's K3V2 result is stated for a packed
 * cache without an fp16 recent-key buffer, which names such a buffer as an
 * option of the serving path). Reading adopted: the keys and values of the R
 * most recent tokens of a sequence stay exactly as appended; a token is
 * quantized with the layer's plan, exactly as without a window, once R newer
 * tokens follow it (tokens leave in order). After T appended tokens the
 * packed cache holds tokens [0, T - w) and the window tokens [T - w, T),
 * w = min(R, T), whatever the sizes of the appends. Decode attends over the
 * packed and the window tokens together.
 *
 * Window buffer (one per sequence, caller-owned, >= kvq_window_bytes(cfg, R)
 * bytes, 16-byte aligned): a ring of R slots, token t in slot t mod R; keys
 * fp32 [R][n_kv_heads][128], then values fp32 [R][n_kv_heads][128] (the
 * appended 16-bit values held exactly in fp32). wlen_dev: int32 [batch],
 * tokens in each window, zero-filled with the buffers; len_dev counts the
 * packed tokens only.
 *
 * kvq_window_append: appends n_new tokens per sequence (k_dev, v_dev as for
 *   kvq_quantize_append). The oldest max(0, wlen + n_new - R) of the window
 *   and new tokens are quantize-appended to the packed cache at len..., the
 *   others enter the ring; then len += evicted, wlen = min(R, wlen + n_new).
 *   A sequence whose evictions do not fit min(cap_tokens) flags CAPACITY and
 *   is left unchanged. R = 0 is kvq_quantize_append (every token quantized,
 *   wlen untouched). Two launches; no workspace.
 * kvq_decode_attn_window: kvq_decode_attn over the packed tokens (len_dev,
 *   max_len >= every len) and the window tokens (wlen_dev) together: one
 *   partial decode of the packed tokens, the records of the window tokens
 *   (fp32 logits q.k log2(e)/sqrt(128) and values rotated like the packed
 *   ones; up to 32 parts of the window per KV head and sequence, in
 *   parallel), one combine; three launches. ws_dev: >=
 *   kvq_window_decode_workspace_bytes(...) bytes, 16-byte aligned,
 *   zero-filled once, reuse rules of kvq_decode_attn; its first
 *   33 batch n_q_heads 132 floats (rounded up to 256 bytes) hold the
 *   records, the rest serves the partial decode.
 * Both return KVQ_OK or a negative code.
 */
KVQ_API size_t kvq_window_bytes(const kvq_cfg* cfg, int R);
KVQ_API int kvq_window_append(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                              const void* v_dev, int kv_dtype, int n_new, void* const* cache_dev,
                              int32_t* len_dev, int64_t cap_tokens, void* const* win_dev,
                              int32_t* wlen_dev, int R, int batch, uint32_t* status_dev,
                              kvq_stream_t stream);
KVQ_API size_t kvq_window_decode_workspace_bytes(const kvq_cfg* cfg, int batch, int n_q_heads,
                                                 int64_t max_len);
KVQ_API int kvq_decode_attn_window(const kvq_cfg* cfg, const void* const* plans_dev,
                                   const void* const* cache_dev, const int32_t* len_dev,
                                   const void* const* win_dev, const int32_t* wlen_dev, int R,
                                   int batch, int64_t max_len, const void* q_dev, int q_dtype,
                                   int n_q_heads, float* out_dev, void* ws_dev, size_t ws_bytes,
                                   uint32_t* status_dev, kvq_stream_t stream);

/*
 * A serving step with the recent-token window: kvq_window_append of n_new
 * tokens per sequence, then kvq_decode_attn_window, with the same results
 * (outputs to fp32 rounding). For 1 <= n_new <= min(R, 64) it is one launch
 * of the decode kernel: the CTAs that own the tiles of the tokens leaving
 * the window quantize-append them (read from their ring slots) and then
 * write the new tokens that take those slots; the CTA that owns the last
 * packed tile writes the new tokens that take free slots; the window's
 * older tokens (from the ring) and the new ones (from k_dev, v_dev) are
 * attended in chunks of 8 by a few CTAs after their tiles, each chunk's
 * record merged with the CTA's own; the last CTA of the sequence to read
 * the lengths writes len += evicted and wlen = min(R, wlen + n_new). Other
 * n_new (or R = 0) run the two calls.
 * Arguments as for those calls; the evictions must fit min(cap_tokens,
 * max_len) (else CAPACITY and the sequence's window is left as it was).
 * step_flags: KVQ_STEP_EARLY as for kvq_append_decode (the previous kernel on
 * the stream then writes neither the caches, the lengths nor the rings);
 * KVQ_STEP_ROPE is refused (the window holds the keys as given).
 * ws_dev: >= kvq_window_decode_workspace_bytes(...) bytes, rules as for
 * kvq_decode_attn_window; the fused and the two-call forms may alternate
 * on one workspace.
 */
KVQ_API int kvq_append_decode_window(const kvq_cfg* cfg, const void* const* plans_dev,
                                     const void* k_dev, const void* v_dev, int kv_dtype,
                                     int n_new, void* const* cache_dev, int32_t* len_dev,
                                     int64_t cap_tokens, void* const* win_dev, int32_t* wlen_dev,
                                     int R, int batch, int64_t max_len, const void* q_dev,
                                     int q_dtype, int n_q_heads, float* out_dev, void* ws_dev,
                                     size_t ws_bytes, int step_flags, uint32_t* status_dev,
                                     kvq_stream_t stream);

/*
 * One serving step in one launch: kvq_quantize_append of n_new tokens per
 * sequence followed by kvq_decode_attn over the grown caches (the pages'
 * packed-cache serving path: append the step's keys and values, then decode).
 * The CTA that owns a new token's tile quantizes and packs it before it
 * streams the tile; every CTA decodes over len + n_new tokens; the last CTA
 * of a sequence to read its length writes len + n_new.
 * Arguments as for the two calls; n_new in 0..64 (k_dev, v_dev:
 * [batch][n_new][n_kv_heads][128] of kv_dtype). A sequence with
 * len + n_new > min(cap_tokens, max_len) gets no append (CAPACITY; len
 * unchanged) and is decoded over its min(len, max_len) tokens. The workspace
 * follows the rules of kvq_decode_attn.
 * The kernel uses programmatic dependent launch: work that reads nothing the
 * previous kernel on the stream writes (the plan, the lookup tables) starts
 * before that kernel ends. step_flags:
 *   KVQ_STEP_EARLY  the lengths are read and the first cache tiles streamed
 *                   before the previous kernel on the stream has finished.
 *                   Only set it when that kernel writes neither these caches
 *                   nor these lengths (e.g. in a loop over layers, where the
 *                   previous kernel is another layer's step, which may share
 *                   the workspace); q, k_dev, v_dev, out and the rest of the
 *                   workspace are always read and written after it (q is
 *                   only prefetched into L2 before it, which reads no value).
 *   KVQ_STEP_ROPE   k_dev holds pre-RoPE keys, rotated to their cache
 *                   positions with base rope_base exactly as by
 *                   kvq_quantize_append_rope (rope_base is ignored without
 *                   this flag).
 * Returns KVQ_OK or a negative code.
 */
KVQ_API int kvq_append_decode(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                              const void* v_dev, int kv_dtype, int n_new, void* const* cache_dev,
                              int32_t* len_dev, int64_t cap_tokens, int batch, int64_t max_len,
                              const void* q_dev, int q_dtype, int n_q_heads, float* out_dev,
                              void* ws_dev, size_t ws_bytes, int step_flags, double rope_base,
                              uint32_t* status_dev, kvq_stream_t stream);

/*
 * Paged caches (no counterpart in the pages, which keep one cache per
 * sequence): the tiles of all sequences live in pages of one pool and a
 * block table says which page holds which span of each sequence, so
 * sequences grow page by page without reserving their full capacity.
 * A page holds page_tiles consecutive 32-token tiles of one sequence for all
 * KV heads, laid out exactly like a contiguous cache of page_tiles tiles
 * (record of tile t, head h of the page at (t n_kv_heads + h) tile_bytes);
 * tile t of sequence b is tile t mod page_tiles of page
 * block_table[b][t / page_tiles]. Codes, norms and decode results are those
 * of a contiguous cache holding the same tokens.
 *
 * pool:        device, 16-byte aligned; page g at pool + g kvq_page_bytes.
 * block_table: device int32 [batch][max_pages]; entries that a call reaches
 *              (tiles below len + n_new) must be page ids in [0, n_pages);
 *              others are never read. An id outside the pool, or a tile past
 *              the row, flags BAD_PAGE: appends skip that tile, decode
 *              streams placeholder bytes instead and its output is invalid.
 *              Pages of different sequences must not overlap.
 * n_pages:     pages in the pool. page_tiles: a power of two, 1..2^20.
 * max_pages:   row length; a sequence holds at most
 *              max_pages * page_tiles * 32 tokens (the capacity that
 *              cap_tokens gives for contiguous caches; at most 2^31 - 1).
 * The block table is read by the kernels as the lengths are: with
 * KVQ_STEP_EARLY it must not be written by the previous kernel on the stream.
 * The library only reads the pool through the table and never allocates or
 * frees pages; the caller owns the pool, the table and the page bookkeeping.
 * Errors (before any launch): KVQ_ERR_ARG for a null page description, pool
 * or block table, a pool off a 16-byte boundary, page_tiles not a power of
 * two in 1..2^20, max_pages or n_pages < 1, or a row capacity above
 * 2^31 - 1 tokens; the other arguments are checked as for the contiguous
 * calls.
 */
typedef struct kvq_pages {
  void* pool;
  const int32_t* block_table;
  int64_t n_pages;
  int32_t page_tiles;
  int32_t max_pages;
} kvq_pages;

/* Bytes of one page (page_tiles * n_kv_heads * kvq_tile_bytes); 0 if invalid. */
KVQ_API size_t kvq_page_bytes(const kvq_cfg* cfg, int32_t page_tiles);

/* kvq_quantize_append into paged caches. rope_base = 0: k_dev holds post-RoPE
 * keys; rope_base > 1: pre-RoPE keys rotated as by kvq_quantize_append_rope. */
KVQ_API int kvq_paged_quantize_append(const kvq_cfg* cfg, const void* const* plans_dev,
                                      const void* k_dev, const void* v_dev, int dtype, int batch,
                                      int n_new, const kvq_pages* pages, int32_t* len_dev,
                                      double rope_base, uint32_t* status_dev,
                                      kvq_stream_t stream);
/* kvq_decode_attn over paged caches (same workspace rules). */
KVQ_API int kvq_paged_decode_attn(const kvq_cfg* cfg, const void* const* plans_dev,
                                  const kvq_pages* pages, const int32_t* len_dev, int batch,
                                  int64_t max_len, const void* q_dev, int q_dtype, int n_q_heads,
                                  float* out_dev, void* ws_dev, size_t ws_bytes,
                                  uint32_t* status_dev, kvq_stream_t stream);
/* kvq_decode_attn_partial over paged caches (one context shard's records). */
KVQ_API int kvq_paged_decode_attn_partial(const kvq_cfg* cfg, const void* const* plans_dev,
                                          const kvq_pages* pages, const int32_t* len_dev,
                                          int batch, int64_t max_len, const void* q_dev,
                                          int q_dtype, int n_q_heads, float* rec_dev,
                                          void* ws_dev, size_t ws_bytes, uint32_t* status_dev,
                                          kvq_stream_t stream);
/* kvq_append_decode over paged caches (capacity from the block table). */
KVQ_API int kvq_paged_append_decode(const kvq_cfg* cfg, const void* const* plans_dev,
                                    const void* k_dev, const void* v_dev, int kv_dtype, int n_new,
                                    const kvq_pages* pages, int32_t* len_dev, int batch,
                                    int64_t max_len, const void* q_dev, int q_dtype,
                                    int n_q_heads, float* out_dev, void* ws_dev, size_t ws_bytes,
                                    int step_flags, double rope_base, uint32_t* status_dev,
                                    kvq_stream_t stream);

/*
 * bf16 comparator (not part of the method): split-K decode attention over an
 * unquantized bf16 cache, built like kvq_decode_attn, to measure the packed
 * path against the dense one on the same shapes ("RoPE-Aware Bit Allocation
 * for KV-Cache Quantization", abstract, compares with fp16 FlashAttention2).
 * k_dev, v_dev: bf16 [batch][n_kv_heads][cap_tokens][128], 16-byte aligned.
 * len_dev: int32 [batch], each <= min(max_len, cap_tokens) (larger values
 *        are clamped and flag CAPACITY).
 * q_dev: bf16 [batch][n_q_heads][128], 4-byte aligned; out_dev: fp32
 *        [batch][n_q_heads][128] = softmax(q k^T / sqrt(128)) v per head.
 * ws_dev: >= kvq_bf16_decode_workspace_bytes(...) bytes, 16-byte aligned,
 *        zero-filled once; same reuse rules as kvq_decode_attn (here only
 *        the merge counters at the end must start at zero).
 * Returns KVQ_OK or a negative code.
 */
KVQ_API size_t kvq_bf16_decode_workspace_bytes(int batch, int n_kv_heads, int n_q_heads,
                                               int64_t max_len);
KVQ_API int kvq_bf16_decode_attn(const void* k_dev, const void* v_dev, const int32_t* len_dev,
                                 int batch, int n_kv_heads, int64_t cap_tokens, int64_t max_len,
                                 const void* q_dev, int n_q_heads, float* out_dev, void* ws_dev,
                                 size_t ws_bytes, uint32_t* status_dev, kvq_stream_t stream);

/*
 * Decode attention without a caller workspace. The paper has no counterpart:
 * this is a library convenience. Same computation, arguments and results as
 * kvq_decode_attn, minus ws_dev / ws_bytes.
 *
 * Who needs it: callers that cannot allocate device memory where they decode
 * - a serving loop being recorded into a CUDA graph (cudaMalloc cannot be
 * captured), an application whose device memory all belongs to a pool this
 * library cannot reach, or code that must not risk the device-wide
 * synchronization cudaMalloc / cudaFree can cause mid-step. The caller still
 * passes every input and output buffer.
 *
 * Scratch: the split partials go to a fixed array of
 * kvq_decode_noalloc_scratch_bytes() (16 MiB) in the library's own device
 * memory, present on every GPU that loads the library until the process
 * exits. A call whose workspace would not fit (kvq_decode_workspace_bytes of
 * the same arguments > 16 MiB; on a B200 that is more than about 100
 * sequences x KV heads) returns KVQ_ERR_WORKSPACE and launches nothing.
 * The call allocates nothing: no cudaMalloc, cudaFree or allocating routine.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture on the device. The cached address
 * belongs to the device's current primary context: after cudaDeviceReset
 * (or anything else that destroys that context) it is stale, and the call
 * must not be used again in the process.
 *
 * Sharing: every call uses the same array, which keeps the last call's
 * contents. The array is laid out like a kvq_decode_attn workspace: split
 * records from its start (always written before they are read) and, at
 * fixed distances from its end, one block per (sequence, KV head) of arrival
 * counters and exponent buckets that must be zero when a call starts. The
 * array is zero when the library is loaded, every completed call clears the
 * blocks it used, and no call's records reach the blocks of another call
 * that fits, so calls of any shapes that fit may follow one another. Calls
 * that overlap on the GPU - on different streams, or from different host
 * threads without ordering - race on the array and may give wrong outputs;
 * order them on one stream.
 */
KVQ_API int kvq_decode_attn_noalloc(const kvq_cfg* cfg, const void* const* plans_dev,
                                    const void* const* cache_dev, const int32_t* len_dev,
                                    int batch, int64_t max_len, const void* q_dev, int q_dtype,
                                    int n_q_heads, float* out_dev, uint32_t* status_dev,
                                    kvq_stream_t stream);

/* Size of the fixed scratch used by kvq_decode_attn_noalloc (16 MiB). */
KVQ_API size_t kvq_decode_noalloc_scratch_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
