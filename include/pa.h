/*
 * pa.h -- C ABI of libpa_b200.so: single-token decode attention over a
 * paged KV cache, and the slot-mapped append of each step's new K/V token,
 * for NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages' statement of the problem, which names
 * them without a formula (miniVLLM docs index, "What is miniVLLM?": paged
 * attention for decode, a paged KV cache; "Explore by topic": fixed-size
 * pages, online softmax; tiny-vllm write-up, "Chi tiet": KV cache,
 * FlashAttention-style online softmax, PagedAttention).  Written out:
 *
 *   for sequence b, query head h, kv head g = h / (Hq / Hkv):
 *     K_t = k_cache[block_tables[b][t / bs]][g][t % bs][:]      (V_t likewise)
 *     s_t = scale * dot(q[b][h], K_t)              for t < context_lens[b]
 *     out[b][h] = sum_t softmax(s)_t * V_t        (bf16, round-to-nearest-even)
 *
 * computed with fp32 products, sums and online-softmax state.
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers on the current CUDA device, owned
 *     by the caller; the library never frees or keeps them.  bf16 tensors
 *     are raw 2-byte values; all are dense, row-major, with the shapes below.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and never synchronise or allocate.
 *   - Host-side checks (NULL pointers, sizes, alignment, supported shapes)
 *     return a negative pa_status and launch nothing.
 *   - Device-side checks (block ids, context lengths, slots) cannot be made
 *     on the host without a sync; a violation sets a bit in the device
 *     error word (PA_DEVERR_*), read with pa_device_errors().  The kernel
 *     never reads or writes out of bounds and never traps; outputs of a call
 *     that set an error bit are unspecified.
 *
 * Layouts:
 *   q, out           [B][Hq][D] bf16
 *   k_cache, v_cache [NB][Hkv][bs][D] bf16: one (block, kv head) tile is
 *                    bs contiguous rows of D values (bs*D*2 bytes)
 *   block_tables     [B][M] int32; entries past ceil(context_len/bs) are
 *                    never read
 *   context_lens     [B] int32, 0 <= L_b <= M*bs (L_b = 0 gives out = 0);
 *                    decode needs NB >= 1 when B > 0
 *   k_new, v_new     [T][Hkv][D] bf16
 *   slot_mapping     [T] int32; slot s writes block s / bs, row s % bs;
 *                    s < 0 marks padding and is skipped
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_NULL = -1,         /* a required pointer is NULL */
    PA_ERR_SHAPE = -2,        /* a size is negative, zero where it must not be, or inconsistent */
    PA_ERR_UNSUPPORTED = -3,  /* head_dim / block_size / GQA group not built into this library */
    PA_ERR_ALIGN = -4,        /* a tensor pointer is not 16-byte aligned */
    PA_ERR_WORKSPACE = -5,    /* workspace NULL or smaller than pa_decode_workspace_bytes() */
    PA_ERR_CUDA = -6,         /* a CUDA runtime call failed (launch, attribute, device query) */
    PA_ERR_SCRATCH_LIMIT = -7 /* pa_decode_static_ws: the problem needs more scratch than
                                 PA_STATIC_SCRATCH_BYTES */
} pa_status;

/* Bits of the device error word. */
#define PA_DEVERR_BLOCK_ID 0x1  /* a block id inside a context was outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT 0x2   /* a context_len was outside [0, max_blocks_per_seq*block_size] */
#define PA_DEVERR_SLOT 0x4      /* an append slot was >= num_blocks*block_size */
#define PA_DEVERR_TIMEOUT 0x8   /* a bounded pipeline wait gave up (internal error) */
#define PA_DEVERR_PREFIX 0x10   /* pa_decode_shared_prefix: a group broke its contract (see there) */

typedef struct pa_dims {
    int32_t num_seqs;           /* B */
    int32_t num_q_heads;        /* Hq, a multiple of Hkv */
    int32_t num_kv_heads;       /* Hkv */
    int32_t head_dim;           /* D */
    int32_t block_size;         /* bs, tokens per physical block */
    int32_t num_blocks;         /* NB, physical blocks in the pool */
    int32_t max_blocks_per_seq; /* M, width of a block_tables row */
} pa_dims;

/*
 * Slot-mapped append ("reshape_and_cache"): for every t < num_tokens with
 * s = slot_mapping[t] >= 0 and every kv head g,
 *     k_cache[s / bs][g][s % bs][:] = k_new[t][g][:]    (v likewise),
 * a bit-exact copy.  Used by decode to store the token being generated
 * before attending over it (a KV-caching engine, miniVLLM review, "What
 * main.py actually does").  Uses dims->num_kv_heads, head_dim, block_size,
 * num_blocks; D must be a multiple of 8.  Slots >= NB*bs are skipped and
 * set PA_DEVERR_SLOT.  Two tokens mapped to one slot: which one lands is
 * unspecified.
 */
PA_API pa_status pa_cache_append(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                          int32_t num_tokens, void* k_cache, void* v_cache,
                          const pa_dims* dims, void* stream);

/*
 * Device workspace pa_decode needs, in bytes, when it runs on `num_ctas`
 * CTAs (0 = the default grid pa_decode picks on the current device).  The
 * workspace holds split-KV partial outputs (two slots per CTA), one merge
 * counter per (sequence, kv head) and the counters of the merge's first
 * level.  It must be zero-filled once before its first use; every completed
 * call leaves it ready for the next (the counters return to zero).  Calls
 * that share one workspace must not overlap on the GPU.  Returns 0 for
 * invalid dims.
 */
PA_API size_t pa_decode_workspace_bytes(const pa_dims* dims, int32_t num_ctas);

/* Grid size (CTAs) pa_decode uses on the current device; <= 0 on error. */
PA_API int32_t pa_decode_default_ctas(void);

/*
 * Paged decode attention (formula at the top of this file).  One persistent
 * CTA per SM walks an equal share of all (sequence, kv-head group, page)
 * work; a staged page holds one block's K and V tiles of up to 8 kv heads,
 * one warp per kv head, and all GQA query heads of a kv head share its
 * tiles.  A sequence whose pages are shared between CTAs is finished by
 * split-KV partials (flash-decoding) and a log-sum-exp merge done by the
 * last CTA to finish its part (in two levels beyond 16 parts).  Supported:
 * block_size 16, head_dim 64 or 128, Hq/Hkv in {1, 2, 4, 8}; fewer than
 * 2^31 cache rows (NB*Hkv*bs).  q, k_cache, v_cache and out must be 16-byte
 * aligned.  The per-page math runs on the tensor cores (mma.sync, fp32
 * accumulation); setting the environment variable PA_DECODE_MATH=simt
 * before the first call selects the fp32 CUDA core variant instead
 * (head_dim*Hq/Hkv <= 256 only).  Split pieces are merged in a fixed
 * order, whatever order they finish in, so repeated calls on the same
 * inputs give bit-identical outputs.  PA_SEG_WEIGHT_BYTES (read at the first
 * call; default 65536) is the fixed cost of finishing a (sequence, head
 * group) segment, in K+V bytes, that the equal-share split charges: larger
 * values cut short contexts into fewer split pieces.
 */
PA_API pa_status pa_decode(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    void* out, const pa_dims* dims, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * One decode step in one launch: the slot-mapped append of the step's new
 * K/V rows (pa_cache_append) and then paged decode attention over the
 * caches including those rows (pa_decode), fused.  Every CTA writes a slice
 * of the rows to the caches and marks the blocks they go to in a hashed
 * bitmap; what a CTA does before reading a marked block depends on
 * num_tokens:
 *   - up to 256 (a decode step has one per sequence): no CTA waits for
 *     another.  When a block's only new row is token b's, at the last
 *     position of sequence b, the CTA reading it patches that row into its
 *     staged copy of the page (bf16 caches); otherwise it writes the block's
 *     new rows to the caches itself before loading it (the same bytes as the
 *     slice owner).  An ordinary launch.
 *   - more: the CTAs meet at a grid barrier (a cooperative launch, so all
 *     are resident), and a CTA waits there only before its first marked
 *     block.
 * Arguments as for the two calls; the workspace as for pa_decode.  Compared
 * with the two calls it saves the append's launch and its latency
 * (miniVLLM docs index, "What is miniVLLM?": low-latency decode; the append
 * and the decode of one step).  Two tokens mapped to one slot: which lands,
 * and which one a sequence reading that slot sees, is unspecified.  After a
 * call that set PA_DEVERR_TIMEOUT the workspace must be zero-filled again.
 */
PA_API pa_status pa_append_decode(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                  int32_t num_tokens, const void* q, void* k_cache, void* v_cache,
                                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                                  void* out, const pa_dims* dims, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * Test hook: pa_decode on exactly `num_ctas` CTAs (1 .. 1024; it decides
 * where contexts are split), that also records every per-CTA segment it computes:
 * segment i covers tokens [t0, t1) of kv head g of sequence b and stores
 *     seg_meta[i] = {b, g, t0, t1}                       int32[capacity][4]
 *     seg_o[i][j][:]  normalised partial output          f32[capacity][G][D]
 *     seg_m[i][j]     max logit (natural-log units)      f32[capacity][G]
 *     seg_l[i][j]     sum_t exp(s_t - seg_m[i][j])       f32[capacity][G]
 * for the G = Hq/Hkv query heads j of kv head g.  *seg_count (device,
 * zeroed by the caller) receives the number of segments; entries past
 * `capacity` are dropped.  `out` is computed as by pa_decode.  The
 * workspace must be sized with pa_decode_workspace_bytes(dims, num_ctas).
 */
PA_API pa_status pa_decode_partials(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             float scale, void* out, const pa_dims* dims, int32_t num_ctas,
                             void* workspace, size_t workspace_bytes, int32_t capacity,
                             int32_t* seg_meta, float* seg_o, float* seg_m, float* seg_l,
                             int32_t* seg_count, void* stream);

/*
 * Allocation-free decode.  No counterpart in the pages: this entry point
 * exists for callers that cannot allocate device memory at the point where
 * they decode -- for example code running inside a host runtime or plugin
 * that owns every device allocation and offers no allocator, or a latency-
 * critical loop where cudaMalloc (which may block and synchronise the
 * device) is not acceptable.  It computes exactly what pa_decode computes,
 * with the same arguments minus the workspace: its scratch (merge counters
 * and split-KV partials) lives in a fixed array of PA_STATIC_SCRATCH_BYTES
 * bytes inside the library, which every GPU that loads the library holds
 * until the process exits.
 *   - Nothing is allocated: no cudaMalloc/cudaFree, no allocating library call.
 *   - A problem whose scratch (pa_decode_workspace_bytes(dims, 0)) exceeds
 *     PA_STATIC_SCRATCH_BYTES is rejected with PA_ERR_SCRATCH_LIMIT before
 *     anything is launched.  The scratch is two partial slots per CTA (one
 *     CTA per SM) of min(Hkv, 8) * Hq/Hkv * head_dim fp32 values, plus 4
 *     bytes per (sequence, kv head): on a 148-SM B200 the largest head shape
 *     built (8 kv heads x a GQA group of 8, head_dim 128) takes 9.9 MB, so
 *     every supported head shape fits with up to 1.7 million (sequence, kv
 *     head) pairs (e.g. 200,000 sequences of 8 kv heads).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents; each call clears the merge counters it needs (an
 *     asynchronous memset on `stream`) before its kernel.  Calls that can
 *     overlap on the GPU (different streams without ordering) race on the
 *     array and give undefined results: order them.
 */
#define PA_STATIC_SCRATCH_BYTES (16u << 20)
PA_API pa_status pa_decode_static_ws(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, const int32_t* context_lens,
                                     float scale, void* out, const pa_dims* dims, void* stream);

/*
 * Shared-prefix ("cascade") decode: pa_decode (optionally fused with the
 * append, as pa_append_decode) for a batch in which runs of consecutive
 * sequences share the first pages of their contexts, as prefix caching
 * leaves them (miniVLLM docs index, "What is miniVLLM?": a paged KV cache
 * with prefix caching; Mini-SGLang write-up, "Key optimizations": Radix
 * Cache reuse of the KV of a common prefix across requests).  The result
 * is the formula at the top of this file; only the order of the work
 * differs.  Group i is the sequences
 *     b in [group_offsets[i], group_offsets[i+1])
 * whose block_tables rows all begin with the same P_i = group_prefix_pages[i]
 * block ids (whole blocks: P_i*bs tokens).  First the queries of all members
 * attend to the P_i shared pages together, each page read once per group
 * (a dense [members*G x keys] x [keys x D] tcgen05 tensor-core tile), giving
 * split-KV partials; then the decode streams only each member's own pages
 * P_i .. ceil(L_b/bs)-1 and merges the prefix partials by log-sum-exp.
 *   - group_offsets [num_groups+1] and group_prefix_pages [num_groups] are
 *     DEVICE int32 arrays; offsets non-decreasing, 0 <= off[0],
 *     off[num_groups] <= B.  Sequences outside every group, and groups with
 *     P_i = 0, are decoded as by pa_decode.
 *   - max_group_size >= every off[i+1] - off[i] (a host value: it sizes
 *     the grid and the workspace).
 *   - A member with L_b < P_i*bs, or past max_group_size in its group, is
 *     decoded over its whole table and PA_DEVERR_PREFIX is set; so it is
 *     for offsets out of order or range, P_i > M, and a member whose table
 *     does not begin with the group's first member's P_i block ids (the
 *     output of such members is unspecified).
 *   - num_tokens > 0 also appends k_new/v_new at slot_mapping first (as
 *     pa_cache_append): fused into the decode as in pa_append_decode (up to
 *     256 tokens), or inside the prefix pass's launch (more); slots must not
 *     fall in the shared blocks, which the prefix pass reads meanwhile.
 *     num_tokens = 0 skips the append (k_new, v_new, slot_mapping unused).
 *   - Two launches: the prefix pass, then the decode as its programmatic
 *     dependent.  With up to 256 new tokens the decode streams the members'
 *     own pages while the prefix pass runs and waits for the pass only
 *     before it reads the pass's partials; with more, it waits for the pass
 *     before reading any page (the pass wrote the new rows).
 *   - Supported shapes and alignment as for pa_decode.  The workspace must
 *     be at least pa_decode_shared_prefix_workspace_bytes(dims, num_groups,
 *     max_group_size) bytes, zero-filled before its first use, and is left
 *     ready for the next call; calls that share it must not overlap.
 *   - The prefix pass splits each group's shared pages into key ranges
 *     (enough CTAs for half a wave; PA_PREFIX_SPLITS=n, 1..16, read at the
 *     first call, overrides); the decode folds one partial per range.  The
 *     decode CTAs that start on the SMs the pass leaves free take a larger
 *     share of the members' own pages (sized by the longest prefix); the
 *     result does not depend on the shares.
 *   - num_groups = 0 is pa_decode / pa_append_decode with this workspace.
 */
PA_API size_t pa_decode_shared_prefix_workspace_bytes(const pa_dims* dims, int32_t num_groups,
                                                      int32_t max_group_size);
PA_API pa_status pa_decode_shared_prefix(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                         int32_t num_tokens, const void* q, void* k_cache, void* v_cache,
                                         const int32_t* block_tables, const int32_t* context_lens, float scale,
                                         const int32_t* group_offsets, const int32_t* group_prefix_pages,
                                         int32_t num_groups, int32_t max_group_size, void* out,
                                         const pa_dims* dims, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * fp8 KV cache (OCP FP8 E4M3 codes with one scale per kv head for K and one
 * for V; the pages' quantization theme applied to the KV cache, MiniVLLM
 * write-up, "量化层" / "量化支持").  A cached value is e4m3(code) * scale[g]:
 *   k_cache [NB][Hkv][16][D] uint8   token-major, as the bf16 cache;
 *   v_cache [NB][Hkv][D][16] uint8   each (block, kv head) tile transposed:
 *            row d holds the 16 tokens' codes of column d, token t at byte
 *            4*((t % 8) / 2) + 2*(t / 8) + t % 2 of the row;
 *   k_scale, v_scale [Hkv] float32 (device).  block_size must be 16.
 * Half the bytes of the bf16 cache per token; the decode is the formula at
 * the top of this file on the dequantized values.
 *
 * pa_cache_append_fp8: the slot-mapped append (as pa_cache_append) of bf16
 * rows, each value encoded as the E4M3 code nearest to x / scale[g] (an
 * IEEE fp32 division; ties to even; magnitudes beyond 448 saturate to 448).
 * D must be a multiple of 8.
 *
 * pa_decode_fp8: pa_decode over fp8 caches (tensor-core policy; head_dim 64
 * or 128, Hq/Hkv in {1, 2, 4, 8}).  q is bf16 and is converted to f16 for
 * the products, so |q| must stay below 65504; softmax state and sums are
 * fp32.  Workspace as for pa_decode (pa_decode_workspace_bytes).
 */
PA_API pa_status pa_cache_append_fp8(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                     int32_t num_tokens, void* k_cache, void* v_cache, const float* k_scale,
                                     const float* v_scale, const pa_dims* dims, void* stream);
PA_API pa_status pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                               const float* v_scale, const int32_t* block_tables, const int32_t* context_lens,
                               float scale, void* out, const pa_dims* dims, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * One fp8 decode step in one launch: pa_cache_append_fp8 of the step's new
 * bf16 rows into the fp8 caches, then pa_decode_fp8 over the caches
 * including them, fused as pa_append_decode fuses the bf16 calls (up to 256
 * tokens: a CTA writes the encoded new rows of a block to the caches itself
 * before loading it; more: a grid barrier of a cooperative launch).
 * Arguments, codes and results as for the two calls; the workspace as for
 * pa_decode.  Graph-capturable like every call here (no allocation, no
 * synchronisation).  After a call that set PA_DEVERR_TIMEOUT the workspace
 * must be zero-filled again.
 */
PA_API pa_status pa_append_decode_fp8(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                      int32_t num_tokens, const void* q, void* k_cache, void* v_cache,
                                      const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                      const int32_t* context_lens, float scale, void* out, const pa_dims* dims,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Multi-query (chunked prefill) attention over the paged cache, the step
 * beside decode in the pages' engines (miniVLLM docs index, "What is
 * miniVLLM?": flash attention for prefill; Mini-SGLang write-up, "Key
 * optimizations": chunked prefill).  Sequence b brings
 * q_len_b = cu_q_lens[b+1] - cu_q_lens[b] query tokens, rows cu_q_lens[b] ..
 * cu_q_lens[b+1]-1 of q [total][Hq][D] (bf16), which are the LAST q_len_b of
 * its context_lens[b] cached tokens (append their K/V rows first, e.g. with
 * pa_cache_append).  Query token i, at position p = L_b - q_len_b + i,
 * attends causally to tokens 0 .. p:
 *     out[cu_q_lens[b] + i][h] = sum_{t <= p} softmax_t(scale * q . K_t) V_t
 * (bf16, round to nearest even; fp32 products, sums and softmax state).
 *   - cu_q_lens [B+1] int32 (device), cu_q_lens[0] = 0, non-decreasing;
 *     max_q_len (host) >= every q_len_b (it sizes the grid; rows past it
 *     are not computed).  q_len_b > L_b sets PA_DEVERR_CONTEXT (the
 *     sequence's output is then unspecified).
 *   - Shapes and alignment as for pa_decode (block_size 16, head_dim 64 or
 *     128, Hq/Hkv in {1, 2, 4, 8}); out [total][Hq][D].  No workspace.
 * One CTA per (sequence, 128-row tile, kv head) streams the sequence's
 * pages up to the tile's last position in blocks of 64 keys and computes
 * the tile on the tcgen05 tensor cores (S and O accumulated in tensor
 * memory, P as bf16).  Environment, read at the first call:
 * PA_PREFILL_BN=128 selects blocks of 128 keys (one CTA per SM);
 * PA_PREFILL_MMA=sync selects the warp-level mma.sync kernels (this call
 * and the prefix pass of pa_decode_shared_prefix).
 */
PA_API pa_status pa_prefill(const void* q, const int32_t* cu_q_lens, int32_t max_q_len, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                            float scale, void* out, const pa_dims* dims, void* stream);

/*
 * Test hook for the bounded waits (no counterpart in the pages).  Every wait
 * of the kernels above gives up after a time limit instead of spinning for
 * ever, sets PA_DEVERR_TIMEOUT and lets the kernel return, so that a broken
 * pipeline leaves the GPU usable.  This call makes such waits run out on
 * purpose: one CTA on `stream` waits, with the bounded polling wait of the
 * decode pipeline and then with the sleeping wait of the prefill pipeline,
 * on a shared-memory mbarrier that nothing arrives on, each for `limit_ns`
 * nanoseconds, and returns.  limit_ns must lie in [1000, 1000000000]
 * (else PA_ERR_SHAPE).  Afterwards pa_device_errors() reports
 * PA_DEVERR_TIMEOUT and the device stays usable.
 */
PA_API pa_status pa_test_wait_timeout(int64_t limit_ns, void* stream);

/*
 * Reads (and, if `clear` != 0, resets) the device error word of the
 * current device.  Synchronous: waits for all prior work on the device.
 */
PA_API pa_status pa_device_errors(int32_t* errors_out, int32_t clear);

/* Static, human-readable name of a pa_status value. */
PA_API const char* pa_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
