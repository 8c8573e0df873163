/*
 * sink_attn.h - C ABI of libsinkattn.so: causal grouped-query attention with
 * a learned per-head attention sink, an optional sliding window and optional
 * packed documents (varlen), forward and backward, for NVIDIA B200 (sm_100a).
 *
 * The operation.  Attention sinks are named in "gpt-oss implementation"
 * (Megatron-LM issue 1739), section "Attention Mechanisms / Attention Sinks"
 * (after StreamingLLM), in "Tricks from OpenAI gpt-oss you can use with
 * transformers" ("Flash Attention 3 with support for attention sinks") and
 * in tpu-inference PR 861 (a kernel argument `attention_sink`).  The pages
 * name the sink without writing it out; the reading implemented here is the
 * gpt-oss one: one extra logit s_h per query head joins each row's softmax
 * denominator and carries no value:
 *
 *   l_ij  = scale * q_i . k_j                      (j allowed for row i)
 *   m_i   = max(s_h, max_j l_ij)
 *   out_i = sum_j e^{l_ij - m_i} v_j / (e^{s_h - m_i} + sum_j e^{l_ij - m_i})
 *   lse_i = m_i + ln(e^{s_h - m_i} + sum_j e^{l_ij - m_i})   (sink included)
 *
 * s_h is used as given (it is not multiplied by `scale`); s_h = -INFINITY
 * turns the sink off.  Query head h reads key/value head h / (Hq / Hkv).
 *
 * Allowed keys.  Positions are local to a document.  For doc-local query
 * position i, key j is allowed iff j <= i and, when window > 0, i - j < window
 * (a window of `window` keys including the query itself).  window <= 0 is
 * full causal.  The alternating sliding-window / full-causal layer pattern of
 * "gpt-oss implementation" ("Alternating Sliding-Window Attention Pattern")
 * is the caller choosing `window` per layer.  Documents follow the
 * intra-document masking request in the same issue: no attention crosses a
 * cu_seqlens boundary.
 *
 * Backward (derivative of the above; dout given):
 *   P_ij = e^{l_ij - lse_i}, P_sink,i = e^{s_h - lse_i}, D_i = dout_i . out_i
 *   dS_ij = P_ij (dout_i . v_j - D_i)
 *   dq_i = scale sum_j dS_ij k_j, dk_j = scale sum_{i, h in group} dS_ij q_i,
 *   dv_j = sum_{i, h in group} P_ij dout_i, dsinks_h = -sum_i P_sink,i D_i.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or synchronises, and every call is
 *     asynchronous on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream).
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns an error status and launches nothing.
 *   - Layouts are dense and row-major: q/out/dout/dq [T][Hq][D],
 *     k/v/dk/dv [T][Hkv][D] (bf16), lse [Hq][T] (fp32), sinks/dsinks [Hq]
 *     (fp32), cu_seqlens [batch+1] (int32, device, cu_seqlens[0] = 0,
 *     cu_seqlens[batch] = T, non-decreasing).
 *   - Supported: D = 64; Hq % Hkv == 0 with G = Hq / Hkv a power of two
 *     <= 128; scale finite and > 0; bf16 tensors 16-byte aligned.
 *   - A device-side wait that exceeds its time limit (about one second; it
 *     never happens in a correct build) makes the kernel record an error
 *     code and return instead of hanging; sink_attn_last_device_error()
 *     reads it.
 */
#ifndef SINK_ATTN_H_
#define SINK_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SINK_ATTN_OK = 0,
    SINK_ATTN_ERR_NULL = 1,          /* a required pointer is NULL */
    SINK_ATTN_ERR_SHAPE = 2,         /* inconsistent or negative sizes */
    SINK_ATTN_ERR_ALIGN = 3,         /* a tensor is not 16-byte aligned */
    SINK_ATTN_ERR_UNSUPPORTED = 4,   /* valid, but outside what this library implements */
    SINK_ATTN_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed */
    SINK_ATTN_ERR_DEVICE_TIMEOUT = 6,/* a kernel gave up on a wait (see sink_attn_last_device_error) */
    SINK_ATTN_ERR_WORKSPACE = 7      /* workspace missing or smaller than sink_attn_bwd_workspace_size() */
} sink_attn_status;

typedef struct {
    int batch;        /* B: number of documents (cu_seqlens has batch+1 entries) */
    int max_seqlen;   /* >= every document length; with cu_seqlens == NULL the
                         common length S of every document (T = B * S) */
    int total_tokens; /* T */
    int num_q_heads;  /* Hq */
    int num_kv_heads; /* Hkv */
    int head_dim;     /* D (64) */
} sink_attn_dims;

/* Forward.  q [T][Hq][D] bf16, k, v [T][Hkv][D] bf16, sinks [Hq] fp32 (may
 * hold -INFINITY), cu_seqlens int32 [batch+1] on the device or NULL (then
 * every document has length max_seqlen).  Writes out [T][Hq][D] bf16 and
 * lse [Hq][T] fp32 (natural log, sink included).  T = 0 is a no-op.  Runs
 * the kernel sink_attn_fwd_kernel_for() names (two query tiles per CTA). */
sink_attn_status sink_attn_fwd(const sink_attn_dims* dims,
                               const void* q, const void* k, const void* v,
                               const float* sinks, const int* cu_seqlens,
                               int window, float scale,
                               void* out, float* lse, void* stream);

/* Forward on CTA pairs: the same operation, arguments, layouts, ownership
 * and errors as sink_attn_fwd() (the online softmax with the sink logit as
 * the first reference max, "Tricks from OpenAI gpt-oss you can use with
 * transformers", kernels section; the window and document masks of "gpt-oss
 * implementation", alternating sliding-window pattern), computed by a kernel
 * launched as clusters of two CTAs whose tensor-core MMAs run on the CTA
 * pair (M = 256 rows: two adjacent query tiles of one key/value head).  Each
 * CTA loads half of every key and value step, and one thread issues the
 * pair's MMAs.  The two tiles of a pair walk the union of their key ranges,
 * so a row's keys may be split into 64-key steps at other boundaries than
 * in sink_attn_fwd(): the results agree with it to rounding, not bit for
 * bit.  Returns SINK_ATTN_ERR_CUDA if the device cannot run clusters of two
 * CTAs of this kernel. */
sink_attn_status sink_attn_fwd_pair(const sink_attn_dims* dims,
                                    const void* q, const void* k, const void* v,
                                    const float* sinks, const int* cu_seqlens,
                                    int window, float scale,
                                    void* out, float* lse, void* stream);

/* The forward kernels of this library.  All compute the same operation with
 * the same arguments; they differ in how query tiles (128 rows: 128/G tokens
 * x the G query heads of one key/value head) map to CTAs, and their results
 * agree to rounding, not bit for bit, because a row's keys may be split into
 * 64-key steps at other boundaries. */
typedef enum {
    SINK_ATTN_FWD_AUTO = 0,      /* the kernel sink_attn_fwd() picks for the sizes */
    SINK_ATTN_FWD_ONE_TILE = 1,  /* one query tile per CTA; its two softmax warpgroups take alternate
                                    64-key steps and merge at the end */
    SINK_ATTN_FWD_TWO_TILES = 2, /* two adjacent query tiles per CTA, one per softmax warpgroup, sharing
                                    one key/value stream (short key ranges: sliding-window layers) */
    SINK_ATTN_FWD_CTA_PAIR = 3   /* two adjacent query tiles on a pair of CTAs (cluster of two) with
                                    M = 256 tensor-core MMAs, as sink_attn_fwd_pair() */
} sink_attn_fwd_kernel_id;

/* The forward with an explicit kernel (a sink_attn_fwd_kernel_id); arguments,
 * layouts and errors as sink_attn_fwd().  An unknown id returns
 * SINK_ATTN_ERR_UNSUPPORTED before any launch. */
sink_attn_status sink_attn_fwd_with(const sink_attn_dims* dims,
                                    const void* q, const void* k, const void* v,
                                    const float* sinks, const int* cu_seqlens,
                                    int window, float scale,
                                    void* out, float* lse, int kernel, void* stream);

/* The sink_attn_fwd_kernel_id sink_attn_fwd() runs for these sizes and
 * window (never SINK_ATTN_FWD_AUTO), or -1 when the sizes are invalid. */
int sink_attn_fwd_kernel_for(const sink_attn_dims* dims, int window);

/* Bytes of device workspace sink_attn_bwd() needs for these sizes
 * (fp32 dq accumulator, per-row D_i, per-block sink partials, padding).
 * Returns 0 when the sizes are invalid. */
size_t sink_attn_bwd_workspace_size(const sink_attn_dims* dims);

/* Backward.  Inputs as for the forward plus the forward's saved out and lse
 * and the upstream gradient dout [T][Hq][D] bf16.  Writes (overwrites, does
 * not accumulate) dq [T][Hq][D], dk, dv [T][Hkv][D] (bf16) and dsinks [Hq]
 * (fp32).  dsinks is reduced in a fixed order and is bitwise reproducible
 * run to run; dq is summed over key tiles in an fp32 accumulator by TMA
 * bulk reduce-adds (performed in L2 in whatever order the tiles finish), so
 * it may differ in the last bits between runs.  `workspace` is caller-owned
 * device memory of at least sink_attn_bwd_workspace_size(dims) bytes,
 * 256-byte aligned; its contents on entry do not matter. */
sink_attn_status sink_attn_bwd(const sink_attn_dims* dims,
                               const void* q, const void* k, const void* v,
                               const float* sinks, const int* cu_seqlens,
                               int window, float scale,
                               const void* out, const float* lse, const void* dout,
                               void* dq, void* dk, void* dv, float* dsinks,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* Size of the library's built-in backward scratch buffer used by
 * sink_attn_bwd_noalloc(): 32 MiB. */
#define SINK_ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* Backward for callers that cannot allocate device memory.  This entry point
 * is an addition of this library; the pages describe nothing like it.
 *
 * Some callers cannot call cudaMalloc or hand over a workspace: code running
 * inside a memory pool or allocator callback that must not re-enter the
 * allocator, host code that is not allowed to grow device memory after
 * start-up, or a binding whose only way to pass memory is the tensors it
 * already owns.  This entry point computes exactly what sink_attn_bwd()
 * computes, with the same arguments minus the workspace: its scratch (fp32 dq
 * accumulator, D_i, sink partials) lives in a fixed array of
 * SINK_ATTN_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 *  - Sizes whose sink_attn_bwd_workspace_size() exceeds the array are refused
 *    with SINK_ATTN_ERR_WORKSPACE before any launch (at 64 query heads and
 *    head dim 64 that is about 2000 tokens; at 8 query heads about 16000).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before capturing a stream into a CUDA graph.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; the kernels re-initialise everything they read (the dq
 *    accumulator is zeroed each call).  Calls whose execution overlaps on the
 *    GPU (different streams, or different host threads) race on the array and
 *    give wrong results: serialise them. */
sink_attn_status sink_attn_bwd_noalloc(const sink_attn_dims* dims,
                                       const void* q, const void* k, const void* v,
                                       const float* sinks, const int* cu_seqlens,
                                       int window, float scale,
                                       const void* out, const float* lse, const void* dout,
                                       void* dq, void* dk, void* dv, float* dsinks,
                                       void* stream);

/* ------------------------------------------------------------------ decode
 * Decode forward over a key/value cache: a few new tokens per sequence are
 * appended to the cache and their queries attend to everything the cache
 * holds for that sequence, with the same sink, window and causal rules as
 * sink_attn_fwd().  This is the incremental form of the forward the pages use
 * for generation with the alternating sliding-window / full layers
 * ("Tricks from OpenAI gpt-oss you can use with transformers", list item
 * "Dynamic Sliding Window Layer & Cache"); the pages do not describe the
 * cache itself, so its layout is this library's own:
 *
 *   - Sequence b owns cache_capacity (C) slots of k_cache / v_cache, each
 *     slot [Hkv][D] bf16: k_cache, v_cache are [batch][C][Hkv][D].  The token
 *     at position p lives in slot p mod C.  With C >= every sequence length
 *     this is a plain linear cache; a sliding-window layer may keep a ring of
 *     C >= window + new_tokens - 1 slots, which holds every key a new query
 *     can see.  A ring smaller than that loses keys: the kernel then records
 *     device error 0x201 (see sink_attn_device_error) and its output is not
 *     defined.
 *   - cache_seqlens [batch] (int32, device) = L0_b, the tokens of sequence b
 *     in the cache before this call.  The call writes the new tokens at
 *     positions L0_b .. L0_b + new_tokens - 1 (slots mod C) and does not
 *     modify cache_seqlens; the caller advances it by new_tokens.
 *   - New query t of sequence b has position i = L0_b + t and sees key
 *     position j iff j <= i and (window <= 0 or i - j < window).
 */
typedef struct {
    int batch;          /* sequences */
    int new_tokens;     /* Lq >= 1: new tokens per sequence (1 for one-token decode) */
    int cache_capacity; /* C: slots per sequence */
    int max_seqlen;     /* upper bound on L0_b + new_tokens over b (sizes the split grid) */
    int num_q_heads;    /* Hq */
    int num_kv_heads;   /* Hkv */
    int head_dim;       /* D (64) */
} sink_attn_decode_dims;

/* Bytes of device workspace sink_attn_decode() needs (per-split partial
 * results); 0 when the sizes are invalid.  Depends on `window`. */
size_t sink_attn_decode_workspace_size(const sink_attn_decode_dims* dims, int window);

/* Decode.  q [batch][new_tokens][Hq][D] bf16, k_new / v_new
 * [batch][new_tokens][Hkv][D] bf16 (appended to the cache by this call),
 * k_cache / v_cache as above (read and written), cache_seqlens as above,
 * sinks [Hq] fp32.  Writes out [batch][new_tokens][Hq][D] bf16 and
 * lse [Hq][batch * new_tokens] fp32 (natural log, sink included).
 * Supported: D = 64, G = Hq / Hkv a power of two with G * new_tokens <= 64.
 * `workspace`: caller-owned device memory of at least
 * sink_attn_decode_workspace_size(dims, window) bytes, 256-byte aligned.
 * batch = 0 is a no-op.  Launches two or three kernels on `stream` (see
 * sink_attn_decode_launches). */
sink_attn_status sink_attn_decode(const sink_attn_decode_dims* dims,
                                  const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, const int* cache_seqlens,
                                  const float* sinks, int window, float scale,
                                  void* out, float* lse,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Decode over an FP8 (e4m3) cache.  As sink_attn_decode(), except that
 * k_cache / v_cache hold e4m3 codes, one byte per element,
 * [batch][C][Hkv][D], with one dequantisation scale per key/value head:
 * key = code * k_scale[g], value = code * v_scale[g] (k_scale, v_scale:
 * fp32 [Hkv], device, > 0).  The pages list FP8 training recipes (Megatron-LM
 * issue 1739 and its example scripts); this is the place on this path where
 * FP8 pays on B200 at head dim 64: decode is HBM-bound, and e4m3 storage
 * halves the bytes the cache moves.  The kernel widens the codes to fp16
 * (every e4m3 value is exact in fp16) and runs fp16 MMAs, so the queries are
 * converted from bf16 to fp16 for them: a query element beyond the fp16
 * range saturates to +-65504, the one input-range limit of this variant
 * (sink_attn_decode has none).  The call quantises the new tokens' k_new / v_new
 * (bf16) as code = e4m3(x * (1 / scale)), rounded to nearest even and
 * saturated to +-448, into their slots.  The workspace size is that of
 * sink_attn_decode_workspace_size(). */
sink_attn_status sink_attn_decode_e4m3(const sink_attn_decode_dims* dims,
                                       const void* q, const void* k_new, const void* v_new,
                                       void* k_cache, void* v_cache, const int* cache_seqlens,
                                       const float* k_scale, const float* v_scale,
                                       const float* sinks, int window, float scale,
                                       void* out, float* lse,
                                       void* workspace, size_t workspace_bytes,
                                       void* stream);

/* Decode over an FP8 (e4m3) cache with the PV product on the FP8 tensor-core
 * path (tcgen05 kind::f8f6f4).  Arguments, cache layout, quantisation of the
 * new tokens and workspace as for sink_attn_decode_e4m3().  The value codes
 * are read as stored (not widened to fp16), and the unnormalised weights
 * p_j = 2^(x_j - m) of each row (m the kernel's running reference of the
 * row, p_j <= 2^8) are rounded to e4m3 (nearest even, saturating) before
 * the MMA; the row sums use the same rounded weights, so every output row is
 * still a convex combination of its cached values.  The rounding moves each
 * weight by at most 2^-4 of itself (e4m3's 3 mantissa bits; below e4m3's
 * normal range, 2^-6, by at most 2^-10), which bounds the extra error of a
 * row with normalised weights pi_j by
 *   |out - exact| <= 2^-4 sum_j pi_j |v_j - out| + 2^-10 max_j pi_j sum_j |v_j - out|
 *   |lse - exact| <= 2^-4 + 2^-10 max_j pi_j * (keys seen)
 * on top of sink_attn_decode_e4m3's own rounding.  The logits keep the fp16
 * path of sink_attn_decode_e4m3 (keys widened to fp16, queries converted to
 * fp16): e4m3 queries would move every logit by up to 2^-4 of its terms. */
sink_attn_status sink_attn_decode_e4m3_f8pv(const sink_attn_decode_dims* dims,
                                            const void* q, const void* k_new, const void* v_new,
                                            void* k_cache, void* v_cache, const int* cache_seqlens,
                                            const float* k_scale, const float* v_scale,
                                            const float* sinks, int window, float scale,
                                            void* out, float* lse,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);

/* Number of kernels one sink_attn_decode / sink_attn_decode_e4m3 call
 * launches for these sizes and window (0 when batch = 0): append, attend and
 * combine, or only the first two when one CTA per (sequence, key/value head)
 * covers the cache (the attend kernel then finishes the rows itself). */
int sink_attn_decode_launches(const sink_attn_decode_dims* dims, int window);

/* Human-readable name of a status code (static string, never NULL). */
const char* sink_attn_status_string(sink_attn_status s);

/* Synchronises `stream` (a cudaStream_t passed as void*), then returns and
 * clears the device error code that a timed-out wait (or a decode ring too
 * small for its window) recorded on the current device: 0 = none, -1 = the
 * synchronisation or the read failed.  These are the only entry points that
 * synchronise.  sink_attn_device_error is the same function under a shorter
 * name. */
int sink_attn_last_device_error(void* stream);
int sink_attn_device_error(void* stream);

/* Self-test of the bounded device waits (failure detection without a fault):
 * one block waits on mbarriers that nothing completes.  One thread gives up
 * after limit_ns (0 < limit_ns <= 1 s), records error code 0x107 and raises
 * the block's abort flag; a thread of another warp, waiting with ten times
 * that limit, must leave through the flag without recording its own code
 * (0x108).  `out`: device pointer to 4 ints (4-byte aligned), written as
 * {first wait returned true, its microseconds, second wait returned true,
 * its microseconds}.  Asynchronous on `stream`; read the recorded code with
 * sink_attn_device_error().  Returns SINK_ATTN_ERR_ALIGN for a NULL or
 * misaligned `out`, SINK_ATTN_ERR_SHAPE for a limit outside the range. */
sink_attn_status sink_attn_selftest_wait(unsigned long long limit_ns, int* out, void* stream);

/* Profiling aid.  Registers two CUDA events (cudaEvent_t passed as void*)
 * that later calls record on their stream immediately before and after one
 * kernel launch: which = 0 -> the forward kernel of sink_attn_fwd,
 * which = 1 -> the main (tensor-core) kernel of sink_attn_bwd.  Passing NULL
 * events clears the slot.  Process-wide and not thread-safe; the events stay
 * owned by the caller.  Returns SINK_ATTN_ERR_SHAPE for an unknown `which`. */
sink_attn_status sink_attn_profile_events(int which, void* ev_begin, void* ev_end);

/* Number of kernels one sink_attn_fwd / sink_attn_bwd call launches for
 * these sizes (0 when T = 0). */
int sink_attn_fwd_launches(const sink_attn_dims* dims);
int sink_attn_bwd_launches(const sink_attn_dims* dims);

#ifdef __cplusplus
}
#endif

#endif /* SINK_ATTN_H_ */
