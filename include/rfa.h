/*
 * rfa.h -- C ABI of librfa.so: rotary position embedding (RoPE) fused into a
 * FlashAttention-style forward pass, and the DynamicNTK sin/cos table, for
 * one NVIDIA B200 (sm_100a).
 *
 * Conventions for every entry point
 *   - Plain pointers and sizes only.  "dev" pointers are CUDA device memory on
 *     the current device, "host" pointers are ordinary host memory.
 *   - The caller owns every buffer.  The library allocates nothing; scratch
 *     memory is the caller's workspace.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*, NULL = legacy default stream).  Host-side validation happens
 *     synchronously before anything is enqueued: on an error nothing runs.
 *   - Tensors are dense and row-major in the stated layout; there are no
 *     stride arguments and no silent fallback to another code path.
 *   - No C++ exception crosses this boundary.
 *   - Errors found on the device (a wait that timed out, lengths that do not
 *     add up) are recorded in a per-device status word that
 *     rfa_get_device_status() reads and clears.
 */
#ifndef RFA_H_
#define RFA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RFA_API __attribute__((visibility("default")))
#else
#define RFA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RFA_OK = 0,
    RFA_ERR_INVALID_ARG = 1, /* null pointer, bad size, inconsistent lengths */
    RFA_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels cover */
    RFA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    RFA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    RFA_ERR_TIMEOUT = 5      /* a device-side wait gave up (status word only) */
} rfa_status;

/* Output / IO element types.  UNDEFINED is the default of the DynamicNTK
 * parameter and is rejected, as on that operator's page (parameter list:
 * "this default type is not usable").  FP32 is an extension for the sin/cos
 * table only. */
typedef enum { RFA_DT_UNDEFINED = 0, RFA_DT_FP16 = 1, RFA_DT_BF16 = 2, RFA_DT_FP32 = 3 } rfa_dtype;

/* BNSD: q [B, Hq, S, D], k/v [B, Hkv, S, D]  (page "RoPE fused into attention
 *       on Ascend", section 3, input_layout="BNSD").
 * TND : packed sequences, q [T, Hq, D], k/v [T, Hkv, D], T = sum of lengths
 *       (the token-major packing of page "DynamicNTKOperation", inputs). */
typedef enum { RFA_LAYOUT_BNSD = 0, RFA_LAYOUT_TND = 1 } rfa_layout;

/*
 * rfa_rope_sincos -- the DynamicNTK sin/cos table.
 * Page "DynamicNTKOperation", sections computation process, inputs, outputs
 * and constraints: for each batch b (its tokens found through the prefix sums
 * of seqLens), freq = outer(positionIds_b, invFreq_b), emb = cat(freq, freq),
 * sin = sin(emb), cos = cos(emb).
 *
 *   positionIds  dev  int32 [ntokens]            any int32 value
 *   invFreq      dev  fp32  [batch, headSize/2]  documented range [0,1), not enforced
 *   seqLens      dev  int32 [batch]              each > 0, sum == ntokens
 *   batch        1..16
 *   ntokens      1..256000
 *   headSize     multiple of 32, <= 2048
 *   outType      RFA_DT_FP16 | RFA_DT_BF16 | RFA_DT_FP32 (UNDEFINED rejected)
 *   sinOut,cosOut dev [ntokens, headSize] of outType, written in full;
 *                columns j and j+headSize/2 are bit-identical.
 *
 * The angle is position*invFreq taken exactly (the fp32 product plus its
 * rounding error, reduced by 2*pi with the two-constant Cody-Waite scheme);
 * sin/cos of the reduced angle are evaluated in fp32 (max abs error below
 * 2e-6 for angles up to 1e6) and rounded to nearest even.  Positions beyond
 * +-2^24 lose low bits in the int32 -> fp32 conversion.
 * Returns RFA_ERR_INVALID_ARG / RFA_ERR_UNSUPPORTED on host-checkable errors.
 * seqLens lives on the device, so its sum is checked by the kernel: if it is
 * not ntokens (or a length is <= 0) nothing is written and the status word
 * becomes RFA_ERR_INVALID_ARG.
 */
RFA_API rfa_status rfa_rope_sincos(const int32_t* positionIds, const float* invFreq, const int32_t* seqLens,
                           int32_t batch, int32_t ntokens, int32_t headSize, rfa_dtype outType,
                           void* sinOut, void* cosOut, void* stream);

/* Parameters of rfa_rope_apply (plain old data). */
typedef struct {
    int32_t layout;       /* RFA_LAYOUT_TND: x [T, H, D], token t uses table row t;
                             RFA_LAYOUT_BNSD: x [B, H, S, D], token (b, s) uses table row b*S + s */
    int32_t T;            /* TND: tokens (>= 1) */
    int32_t B, S;         /* BNSD: batch, sequence length (>= 1 each) */
    int32_t Hq, Hkv;      /* heads of q and of k (>= 1; 0 when that tensor is not given) */
    int32_t D;            /* head dim: even, multiple of 16, <= 512 */
    int32_t io_dtype;     /* RFA_DT_BF16 | RFA_DT_FP16: q, k, outputs and the cache */
    int32_t table_dtype;  /* RFA_DT_FP16 | RFA_DT_BF16 | RFA_DT_FP32: sin, cos */
    int32_t interleaved;  /* 0: rotate-half pairs (j, j + D/2); 1: adjacent pairs (2i, 2i+1) */
} rfa_rope_apply_params;

/*
 * rfa_rope_apply -- the Rope operator: q, k, sin and cos in, rotated q and k
 * out (page "DynamicNTKOperation", operator context: DynamicNTK outputs sin
 * and cos, which go with q and k into the Rope operator), optionally writing
 * the rotated keys into a KV cache.  For every row x of width D of q and k and
 * its token's table rows:
 *     out[j] = x[j] * cos[j] + rot(x)[j] * sin[j]
 * with rot(x) = (-x[D/2..D), x[0..D/2)) for rotate-half pairs, or
 * rot(x)[2i] = -x[2i+1], rot(x)[2i+1] = x[2i] for adjacent pairs (the
 * (x1,x2),(x3,x4),... blocks of page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE",
 * sec. 6; such tables hold the angle of pair i in columns 2i and 2i+1).
 * Arithmetic in fp32, outputs rounded to nearest even.
 *
 *   q, k          dev  io_dtype [T, Hq|Hkv, D] (TND) or [B, Hq|Hkv, S, D] (BNSD);
 *                 either may be NULL (then its heads must be 0)
 *   sin, cos      dev  table_dtype [T or B*S, D], e.g. rfa_rope_sincos's output
 *   q_out, k_out  dev  like q, k; may equal q, k (in place); k_out may be NULL
 *                 when the rotated keys only go to the cache
 *   cache_slots   dev  int32 [T or B*S] or NULL: token t's rotated keys go to
 *                 k_cache row cache_slots[t]; negative slots are skipped
 *   k_cache       dev  io_dtype [cache_rows, Hkv, D] (NULL iff cache_slots NULL)
 *   cache_rows    rows of k_cache; a slot >= cache_rows is not written and the
 *                 status word becomes RFA_ERR_INVALID_ARG
 * Pointers 16-byte aligned.  Returns RFA_ERR_INVALID_ARG for null/misaligned
 * pointers or bad sizes, RFA_ERR_UNSUPPORTED for other dtypes.
 */
RFA_API rfa_status rfa_rope_apply(const rfa_rope_apply_params* p, const void* q, const void* k, const void* sin,
                                  const void* cos, void* q_out, void* k_out, const int32_t* cache_slots,
                                  void* k_cache, int64_t cache_rows, void* stream);

/* Parameters of rfa_kv_rms_norm_rope_cache (plain old data). */
typedef struct {
    int32_t T;            /* tokens (>= 1) */
    int32_t Hkv;          /* kv heads (>= 1) */
    int32_t D;            /* head dim: 16, 32, 64, 128, 256 or 512 */
    int32_t io_dtype;     /* RFA_DT_BF16 | RFA_DT_FP16: k, v and both caches */
    int32_t table_dtype;  /* RFA_DT_FP16 | RFA_DT_BF16 | RFA_DT_FP32: sin, cos */
    int32_t interleaved;  /* 0: rotate-half pairs; 1: adjacent pairs (as rfa_rope_apply) */
    float eps;            /* RMSNorm epsilon, finite and >= 0 */
} rfa_kv_cache_params;

/*
 * rfa_kv_rms_norm_rope_cache -- RMSNorm, RoPE and the KV-cache write in one
 * pass: the kv_rms_norm_rope_cache op of page "RoPE fused into attention on
 * Ascend" (sec. 5.2), which names it without stating its formula; the reading
 * taken: for token t and kv head h,
 *     k_cache[slots[t], h, :] = rope(gamma * k[t,h,:] / sqrt(mean(k[t,h,:]^2) + eps))
 *     v_cache[slots[t], h, :] = v[t,h,:]
 * with RMSNorm as on page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE" (sec. 8) and
 * rope() the Rope operator of rfa_rope_apply on the token's table row.
 * Tokens with slots[t] < 0 are skipped.  Arithmetic in fp32, cache rows
 * rounded to nearest even; v rows are copied bit for bit.
 *
 *   k, v          dev  io_dtype [T, Hkv, D]
 *   gamma         dev  fp32 [D]
 *   sin, cos      dev  table_dtype [T, D]
 *   slots         dev  int32 [T]
 *   k_cache, v_cache dev io_dtype [cache_rows, Hkv, D]
 *   cache_rows    >= 1; a slot >= cache_rows is not written and the status word
 *                 becomes RFA_ERR_INVALID_ARG
 * The caches must not overlap k or v (the rows are read ahead of the cache
 * writes).  Pointers 16-byte aligned (slots 4-byte).  Returns
 * RFA_ERR_INVALID_ARG for null/misaligned pointers or bad sizes.
 */
RFA_API rfa_status rfa_kv_rms_norm_rope_cache(const rfa_kv_cache_params* p, const void* k, const void* v,
                                              const float* gamma, const void* sin, const void* cos,
                                              const int32_t* slots, void* k_cache, void* v_cache,
                                              int64_t cache_rows, void* stream);

/* Parameters of rfa_decode_rope_attention (plain old data). */
typedef struct {
    int32_t B;                /* sequences (>= 1) */
    int32_t Hq, Hkv;          /* query / kv heads; Hq % Hkv == 0, G = Hq / Hkv */
    int32_t Sq;               /* new tokens per sequence (>= 1); G * Sq <= 128 */
    int32_t D;                /* head dim: 64 or 128 */
    int32_t Smax;             /* cache rows per sequence */
    int32_t max_kv_len;       /* bound on kv_lens (Sq..Smax), used to split the keys across CTAs */
    int32_t causal;           /* 1: new token s sees keys [0, kv_len - Sq + s]; 0: all kv_len keys */
    int32_t io_dtype;         /* RFA_DT_BF16 | RFA_DT_FP16: q, caches and out */
    int32_t rope_interleaved; /* 0: rotate-half pairs; 1: adjacent pairs (as the cache was written) */
    float scale;              /* softmax scale; 0 -> 1/sqrt(D) */
    int32_t num_splits;       /* parts each sequence's keys are split into across CTAs (whole
                                 128-key tiles; clamped to the tiles of max_kv_len);
                                 0 -> the library's plan; < 0 -> RFA_ERR_INVALID_ARG */
    double rope_base;         /* invFreq_j = base^(-2j/D) when invFreq is NULL */
} rfa_decode_params;

/*
 * rfa_decode_rope_attention -- a decode step over a KV cache: the Sq new
 * tokens of each sequence attend to its cached keys and values (page "RoPE,
 * RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 12-13: every decode step reads the
 * cached K/V, shared by a group of query heads).  The new queries are rotated
 * in the kernel at their positions; the cached keys are taken as stored (they
 * were rotated when written, e.g. by rfa_rope_apply or
 * rfa_kv_rms_norm_rope_cache with slot = b * Smax + t).  The new tokens are
 * the last Sq of the kv_len cached entries:
 *     out[b,h,s] = softmax_j(rope(q[b,h,s], q_pos[b,s]) . K[b,j,h/G] * scale) V[b,j,h/G]
 * over j in [0, kv_len_b - Sq + s] (causal) or [0, kv_len_b).
 *
 *   q, out        dev io_dtype [B, Hq, Sq, D]
 *   k_cache, v_cache dev io_dtype [B, Smax, Hkv, D]
 *   q_pos         dev int32 [B, Sq]
 *   kv_lens       dev int32 [B]; each in [Sq, max_kv_len], else the status word
 *                 becomes RFA_ERR_INVALID_ARG (the length is clamped)
 *   invFreq       dev fp32 [B, D/2] or NULL (then base^(-2j/D) from rope_base)
 *   workspace     dev, 256-byte aligned, >= rfa_decode_rope_attention_workspace(p)
 *                 bytes (at least 256): when the keys are split across CTAs, the
 *                 fp32 partial results that a second kernel merges (launched as a
 *                 programmatic dependent launch, so it starts as the first ends).
 *                 The queries' cos/sin are formed inside the attention kernel.
 * Returns RFA_ERR_INVALID_ARG / RFA_ERR_UNSUPPORTED / RFA_ERR_WORKSPACE on
 * host-checkable errors; nothing is enqueued then.
 */
RFA_API size_t rfa_decode_rope_attention_workspace(const rfa_decode_params* p);
RFA_API rfa_status rfa_decode_rope_attention(const rfa_decode_params* p, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* q_pos, const int32_t* kv_lens,
                                             const float* invFreq, void* out, void* workspace, size_t ws_bytes,
                                             void* stream);

/* Parameters of rfa_fused_rope_attention (plain old data). */
typedef struct {
    int32_t B;             /* BNSD: batch size; TND: number of packed sequences (1..16) */
    int32_t Hq;            /* query heads (head_num) */
    int32_t Hkv;           /* key/value heads; Hq % Hkv == 0, group G = Hq/Hkv,
                              query head h reads kv head h / G */
    int32_t S;             /* BNSD: sequence length (>= 1); TND: ignored */
    int32_t D;             /* head dim: 64 or 128 */
    int32_t layout;        /* rfa_layout */
    int32_t causal;        /* 1: key index > query index (within a sequence) masked */
    int32_t io_dtype;      /* RFA_DT_BF16 or RFA_DT_FP16 for q, k, v and out */
    float scale;           /* softmax scale; 0 -> 1/sqrt(D) */
    int32_t rope_interleaved; /* 0: rotate-half pairs (i, i + D/2); 1: adjacent pairs
                              (2i, 2i+1), the (x1,x2),(x3,x4),... blocks of page "RoPE,
                              RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 6; pair i turns by
                              position * invFreq_i in both */
    double rope_base;      /* invFreq_j = base^(-2j/D) (page "RoPE fused into
                              attention on Ascend", section 1.2), e.g. 10000 */
    int32_t ntk_enable;    /* dynamic NTK (page "DynamicNTKOperation", function
                              description): for a sequence of length S_b > L the
                              base becomes base*((f*S_b/L)-(f-1))^(D/(D-2)) */
    int32_t ntk_train_len; /* L */
    double ntk_factor;     /* f (rope_scaling_factor) */
} rfa_attn_params;

/* Bytes of device workspace rfa_fused_rope_attention needs for `ntokens`
 * tokens (BNSD: B*S; TND: sum of lengths).  Returns 0 for invalid params. */
RFA_API size_t rfa_fused_rope_attention_workspace(const rfa_attn_params* p, int64_t ntokens);

/*
 * rfa_fused_rope_attention -- out = softmax(Q'K'^T * scale) V with Q' and K'
 * the rotate-half RoPE rotations of q and k (x' = x*cos + rotate_half(x)*sin
 * with cos/sin of cat(freq, freq)), causal or not, GQA.
 * Pages: "RoPE fused into attention on Ascend" (sections 3 and 5: the fused
 * operator; rotated Q/K stay on chip), "FlashAttention in ops-transformer"
 * (tiling, online softmax), "DynamicNTKOperation" (the sin/cos definition and
 * the NTK rule), "RoPE, RMSNorm, GQA/MQA" (section 12, grouped heads).
 *
 *   p          host  parameters (see rfa_attn_params)
 *   q, k, v    dev   io_dtype, layout per p->layout (see rfa_layout)
 *   position   dev   int32, BNSD [B, S] / TND [T]: the position of each token
 *                    (any int32; it only sets the rotation angle)
 *   seqLens_host host int32 [B], TND only (each > 0); NULL for BNSD
 *   invFreq    dev   fp32 [B, D/2] per-sequence inverse frequencies, or NULL
 *                    to derive them from rope_base (+ NTK) in fp64 on the host,
 *                    rounded once to fp32
 *   out        dev   io_dtype, same shape and layout as q
 *   workspace  dev   >= rfa_fused_rope_attention_workspace(p, T) bytes,
 *                    256-byte aligned; holds the cos/sin table of this call
 *                    (T*D*2 bytes: D/2 fp16 cos and D/2 fp16 sin values per
 *                    token), per-sequence angle seeds (784 bytes
 *                    each) -- tables, never rotated Q/K -- and, in its
 *                    last 256 bytes, the attention kernel's two work counters
 * Rotated Q and K exist only in shared memory.  The call enqueues the cos/sin
 * table kernels (which zero the work counters) and the fused attention kernel:
 * a persistent grid of one CTA per SM taking work items from the counters (its
 * last CTA leaves them at zero).  Calls that share a workspace must not
 * overlap on the GPU.
 */
RFA_API rfa_status rfa_fused_rope_attention(const rfa_attn_params* p, const void* q, const void* k, const void* v,
                                    const int32_t* position, const int32_t* seqLens_host,
                                    const float* invFreq, void* out, void* workspace, size_t ws_bytes,
                                    void* stream);

/*
 * The same operation in two steps, for callers that keep the cos/sin table
 * of a batch of positions and reuse it across calls (page "RoPE fused into
 * attention on Ascend", section 6.2: precompute the lookup table once and
 * register it, rather than regenerating the frequencies on every call).
 *
 * rfa_rope_attention_table: writes the cos/sin table of p's tokens into
 *   workspace (same size and alignment rule as above).  Arguments as for
 *   rfa_fused_rope_attention.
 * rfa_fused_rope_attention_with_table: the attention kernel alone, reading a
 *   table that rfa_rope_attention_table wrote for the same p, positions and
 *   seqLens_host.  The table and seeds are only read; the work counters are
 *   used and left at zero, so the table can serve any number of calls, one
 *   after another (calls sharing the workspace must not overlap on the GPU).
 * rfa_fused_rope_attention == rfa_rope_attention_table followed by
 * rfa_fused_rope_attention_with_table on the same stream.
 */
RFA_API rfa_status rfa_rope_attention_table(const rfa_attn_params* p, const int32_t* position,
                                            const int32_t* seqLens_host, const float* invFreq, void* workspace,
                                            size_t ws_bytes, void* stream);
RFA_API rfa_status rfa_fused_rope_attention_with_table(const rfa_attn_params* p, const void* q, const void* k,
                                                       const void* v, const int32_t* seqLens_host, void* out,
                                                       void* workspace, size_t ws_bytes, void* stream);

/*
 * rfa_fused_rope_attention_noalloc -- rfa_fused_rope_attention without a
 * caller-provided workspace, for callers that cannot allocate device memory
 * where they call this library: code running while a stream is captured into
 * a CUDA graph, plugins whose host framework owns every device buffer and
 * passes a kernel only its inputs and outputs, real-time callers that may not
 * block on an allocator.  (The pages have no counterpart; this is a service
 * of this library.)
 *
 * Arguments and results are those of rfa_fused_rope_attention minus
 * workspace/ws_bytes.  The scratch (cos/sin table, recurrence seeds and work
 * counters) is a fixed area of about 16.8 MB inside the library's module, held by every
 * device that loads the library until the process exits.  Limits: at most
 * 65536 tokens (BNSD: B*S), at most 16 sequences (BNSD: batches), D <= 128;
 * larger problems return RFA_ERR_WORKSPACE before anything is enqueued.
 * This entry point allocates nothing.  Its first call on a device looks up the
 * scratch's device address (make that first call before any stream capture).
 * All calls share the one scratch area, which keeps the last call's contents:
 * calls whose work overlaps on the GPU (e.g. on different streams without
 * ordering) race and must be serialised by the caller.
 */
RFA_API rfa_status rfa_fused_rope_attention_noalloc(const rfa_attn_params* p, const void* q, const void* k,
                                                    const void* v, const int32_t* position,
                                                    const int32_t* seqLens_host, const float* invFreq, void* out,
                                                    void* stream);

/* Synchronises `stream`, then returns and clears the current device's status
 * word (RFA_OK if no kernel recorded an error).  RFA_ERR_CUDA if the
 * synchronisation itself failed. */
RFA_API rfa_status rfa_get_device_status(void* stream);

/* Sets, on the current device, how long a kernel role waits for another
 * (an mbarrier phase) before giving up: on expiry the kernel records
 * RFA_ERR_TIMEOUT, its roles stop, its in-flight copies and MMAs are drained
 * (those drains keep their own 2 s limit) and it returns.  0 restores the
 * default of 2 s.  Meant for failure-detection tests, which lower it so that
 * waits run out on purpose; synchronous; must not overlap running kernels of
 * this library.  RFA_ERR_CUDA if the device variable cannot be written. */
RFA_API rfa_status rfa_set_wait_limit_ns(uint64_t ns);

/* Failure-detection switch on the current device, off by default.  While on
 * (nonzero), the attention kernels (fused and decode) publish no work item:
 * each of their roles waits on an item barrier that nothing arrives on, the
 * wait runs out at the limit set by rfa_set_wait_limit_ns, the kernel records
 * RFA_ERR_TIMEOUT, leaves its output unwritten and returns with the context
 * intact.  0 turns it off.  Synchronous; must not overlap running kernels of
 * this library.  RFA_ERR_CUDA if the device variable cannot be written. */
RFA_API rfa_status rfa_set_hold_items(int32_t on);

/* Static, human-readable name of a status code. */
RFA_API const char* rfa_status_string(rfa_status s);

/* Library version as 10000*major + 100*minor + patch. */
RFA_API int32_t rfa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RFA_H_ */
