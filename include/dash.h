/*
 * dash.h -- C ABI of the B200 DashAttention forward-pass library (libdash_b200.so).
 *
 * DashAttention ("DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
 * xllm-io paper review page, section 3 "core formulas"; gist.science technical summary,
 * "Methodology") is three-stage sparse attention:
 *   Stage 0 (Eq. 4)   chunk summaries  kbar_c^(r) = sum_{t in chunk c} softmax_t(<qbar^(r),k_t>/sqrt(d)) k_t
 *   Stage 1 (Eq. 6)   routing          what_i^(h) = alpha-entmax(gamma * <q_i^(h), kbar_c^(r)>/sqrt(d))
 *                     GQA average      w_i^(r) = mean_{h in group r} what_i^(h); routed set R = support
 *   Stage 2 (Prop. 4.1) biased softmax o_i = softmax_j(<q_i,k_j>/sqrt(d) + d_ij) V over the routed
 *                     chunks' tokens and the diagonal tokens c(i)B..i, with
 *                     d_ij = (log w_{i,c(j)} - mean_{c in R} log w_{i,c}) / sigma on routed tokens, 0 on
 *                     the diagonal (equivalent to Eq. 9 with the Eq. 11-12 prior).
 * A query at position i routes over the complete chunks c < floor(i/B); its own chunk is always
 * the diagonal branch.  Head h uses KV head floor(h / (h_q/h_kv)).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated; the caller allocates and owns every
 *     buffer, including the workspace.  The library never allocates, frees or synchronises.
 *   - Every call only enqueues kernels on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream) and returns; results are ready when the stream reaches them.
 *   - Layouts: Q, O [batch, n, h_q, d_h], K, V [batch, n, h_kv, d_h] addressed through element
 *     strides {batch, position, head}; the d_h elements of one head are contiguous.  Element type
 *     is `dtype` (fp32 or bf16).  qbar, kbar and every routing/bias value are fp32.
 *   - Alignment: Q, K, V, O base pointers and strides*sizeof(element) must be multiples of 16
 *     bytes; other pointers 4 bytes.
 *   - Return value: DASH_OK (0) or a negative DASH_E* status.  Arguments are checked before any
 *     launch; on an error nothing is enqueued.  DASH_ELAUNCH reports a failed kernel launch.
 *
 * Environment switches (read once per process; for comparison runs and tests -- every setting
 * computes the same routes and outputs, only the kernels that produce them differ):
 *   DASH_STAGE2=mma       prefill Stage 1 / Stage 2 and decode Stage 2 on the warp-level mma.sync
 *                         kernels instead of the tcgen05 / TMA ones (paged decode keeps the TMA path)
 *   DASH_STAGE2=pair      prefill Stage 2 on the paired-tile tcgen05 kernel (two 128-row tiles per
 *                         block share one walk of 128-key jobs; g in {4, 8, 16}) instead of the
 *                         one-tile kernel (64-key jobs, two blocks per SM)
 *   DASH_CLUSTER=0        prefill Stage 2 forms its 128-row tiles from consecutive positions
 *                         instead of grouping positions with similar routes (the grouping changes
 *                         only the schedule: outputs are bit-identical)
 *   DASH_LONG_ROUTE=off   rows of more than 512 chunks are routed by the per-shape kernels instead
 *                         of the long-row tcgen05 kernel
 *   DASH_DEC_ROUTE=heads  decode Stage 1 runs as three per-head launches instead of one clustered
 *                         launch (the path very long contexts take anyway)
 */
#ifndef DASH_H
#define DASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    DASH_OK = 0,
    DASH_EINVAL = -1,       /* bad shape / hyper-parameter / null required pointer */
    DASH_EUNSUPPORTED = -2, /* valid but not built: d_h, chunk, group size or dtype */
    DASH_EWORKSPACE = -3,   /* workspace smaller than dash_workspace_size() */
    DASH_EALIGN = -4,       /* pointer or stride alignment */
    DASH_ELAUNCH = -5       /* a kernel launch failed (cudaGetLastError) */
};

enum { DASH_F32 = 0, DASH_BF16 = 1 };
enum { DASH_OP_PREFILL = 0, DASH_OP_DECODE = 1, DASH_OP_BACKWARD = 2 };

typedef struct {
    int batch;
    int seqlen;     /* prefill: sequence length n; decode/append: K/V cache capacity (positions) */
    int h_q, h_kv;  /* h_q % h_kv == 0; group size g_q = h_q / h_kv in {1, 2, 4, 8, 16} */
    int d_h;        /* head dimension: 64 or 128 */
    int chunk;      /* B: 1, 16, 32, 64 or 128 (1: every token is its own chunk, Stage 0 is the identity
                       and Stage 1 is entmax over the visible tokens) */
    float alpha;    /* entmax alpha in (1, 2] (section 3 background formula) */
    float gamma;    /* routing scale gamma >= 0 (Eq. 6); 0 routes every visible chunk uniformly */
    float inv_sigma;/* 1/sigma of Eq. 11 / Prop. 4.1; 1 = plain prior, 0 = sigma -> infinity */
    int dtype;      /* DASH_F32 or DASH_BF16 for Q, K, V, O */
    long long q_strides[3], k_strides[3], v_strides[3], o_strides[3]; /* elements: b, pos, head */
} dash_params;

/* Routing lists written by Stage 1 and read by Stage 2 (section 3, Stage 1 kernel: the routed
 * support after the GQA average).  Any pointer may be NULL; the lists then live in the workspace.
 *   counts    int32 [batch, h_kv, n]                |R_i| for KV head r at position i
 *   chunk_idx int32 [batch, h_kv, dash_route_capacity(p)]  routed chunk ids, ascending; row i's
 *             list starts at tri(i) = B*c*(c-1)/2 + (i - c*B)*c with c = floor(i/B)
 *   bias      fp32, same layout as chunk_idx: d_ij of Prop. 4.1 for the listed chunk
 *   bitmask   uint32 [batch, h_kv, n, ceil(T_c/32)] bit c set iff chunk c is routed (the pages'
 *             bit-packed block mask, 32 columns per word); written only when non-NULL. */
typedef struct {
    int* counts;
    int* chunk_idx;
    float* bias;
    uint32_t* bitmask;
} dash_route_out;

/* Bytes of device workspace `op` (DASH_OP_PREFILL or DASH_OP_DECODE) needs for these params;
 * 0 on invalid params.  The workspace must be 256-byte aligned. */
size_t dash_workspace_size(const dash_params* p, int op);

/* Byte offset inside the prefill or decode workspace (op) of an int32 status word: a prefill (its
 * Stage 0) or a decode call clears it, and
 * a kernel whose bounded wait on an on-chip barrier timed out writes a non-zero code there and
 * leaves instead of hanging (read it after the stream has finished).  -1 for invalid params or
 * an op without such a word. */
long long dash_error_word_offset(const dash_params* p, int op);

/* Byte offset inside the prefill workspace of the order in which the tensor-core Stage 2 (the
 * DashAttention review's Stage 2 kernel row) tiles the positions: int32 [batch][h_kv][n], entry k of
 * (b, r) the position in slot k; the tile of 128 query rows numbered t takes the slots
 * t*128/g .. (t+1)*128/g - 1.  Valid after a prefill's Stage 2 has run on the stream (read it after
 * the stream has finished).  -1 when the default Stage 2 keeps the positions in sequence order for
 * these params (no grouping: g other than 8 or 16, another Stage 2 kernel, DASH_CLUSTER=0) or for
 * invalid params.  A diagnostic: it tells which positions shared a tile, i.e. how much work beyond
 * the routed pairs a tile executed. */
long long dash_prefill_order_offset(const dash_params* p);

/* Routing-list entries per (batch, KV head) for prefill: sum over positions of floor(i/B). */
long long dash_route_capacity(const dash_params* p);

/* Causal prefill forward (Stages 0, 1, 2) of Q, K, V [batch, n, *, d_h] into O.
 *   qbar      fp32 [h_kv, d_h]  learned summary query of Eq. 4 (read only)
 *   kbar_out  fp32 [batch, h_kv, floor(n/B), d_h] Stage-0 summaries, or NULL (then in workspace)
 *   route     optional routing outputs (see dash_route_out), or NULL */
int dash_prefill(const dash_params* p, const void* Q, const void* K, const void* V,
                 const float* qbar, void* O, float* kbar_out, const dash_route_out* route,
                 void* workspace, size_t ws_bytes, void* stream);

/* One stage of dash_prefill on its own (same arguments): stage 0 writes the summaries, stage 1
 * reads them and writes the routing lists, stage 2 reads both and writes O.  Running the three
 * stages in order on one stream with the same buffers equals dash_prefill; the intermediate
 * results must stay in kbar_out / route / workspace between the calls.
 * DASH_STAGE2_BITMASK is Stage 2 driven by the bit-packed block mask M_i (route->bitmask, written
 * by a stage-1 call that was given a bitmask output; the paper review's Stage 2 kernel walks the
 * active chunks of M) together with the bias lists, instead of the chunk-id lists; its output
 * equals DASH_STAGE2's bit for bit (same tensor-core kernel, same schedule).  DASH_EINVAL without
 * route->bitmask; DASH_EUNSUPPORTED unless bf16, d_h = 128, chunk 32 / 64 / 128. */
enum { DASH_STAGE0 = 0, DASH_STAGE1 = 1, DASH_STAGE2 = 2, DASH_STAGE2_BITMASK = 3 };
int dash_prefill_stage(const dash_params* p, int stage, const void* Q, const void* K, const void* V,
                       const float* qbar, void* O, float* kbar_out, const dash_route_out* route,
                       void* workspace, size_t ws_bytes, void* stream);

/* Build the summary cache of already-filled K caches (Eq. 4): for each sequence b with length
 * L_b = seqlens[b] (device int32), writes kbar_cache[b, r, c] for every complete chunk
 * c < floor(L_b/B) and the running state of the incomplete chunk into partial_state.
 *   kbar_cache     fp32 [batch, h_kv, floor(seqlen/B), d_h]
 *   partial_state  fp32 [batch, h_kv, d_h + 2]: acc[d_h], running max m, running sum l of the
 *                  online softmax over the incomplete chunk's keys, in base 2: m is the largest
 *                  <qbar,k> log2(e)/sqrt(d_h) so far, l = sum 2^(a - m), acc = sum 2^(a - m) k
 *                  (m = -inf, l = 0, acc = 0 when the chunk is empty); acc / l is the running
 *                  summary */
int dash_summary_build(const dash_params* p, const void* K_cache, const float* qbar,
                       const int* seqlens, float* kbar_cache, float* partial_state, void* stream);

/* Incremental decoding, step 1 of 2: append one token per sequence.  k_new, v_new
 * [batch, h_kv, d_h] (contiguous, dtype) are written at position L_b = seqlens[b] of the caches
 * (k/v strides from p), the incomplete-chunk state is updated with the new key (online softmax of
 * Eq. 4), the chunk's summary is written to kbar_cache when the key completes it (the summary is
 * fixed from then on), and seqlens[b] becomes L_b + 1.  Requires L_b < seqlen. */
int dash_summary_append(const dash_params* p, const void* k_new, const void* v_new,
                        const float* qbar, void* K_cache, void* V_cache, float* kbar_cache,
                        float* partial_state, int* seqlens, void* stream);

/* Incremental decoding, step 2 of 2: the query q [batch, h_q, d_h] (contiguous, dtype) of each
 * sequence sits at position L_b - 1 (L_b = seqlens[b] after the append) and attends over cache
 * positions 0..L_b-1: Stage 1 over the cached summaries of chunks c < floor((L_b-1)/B), then
 * Stage 2 split along the routed chunks, then a log-sum-exp merge.  O [batch, h_q, d_h]
 * (contiguous, dtype).  route: optional, counts [batch, h_kv], chunk_idx / bias
 * [batch, h_kv, floor(seqlen/B)]. */
int dash_decode(const dash_params* p, const void* q, const void* K_cache, const void* V_cache,
                const float* kbar_cache, const int* seqlens, void* O, const dash_route_out* route,
                void* workspace, size_t ws_bytes, void* stream);

/* Paged K/V caches for incremental decoding (a serving layout; the paper's kernels take
 * contiguous caches).  K and V live in pools of pages [num_pages][page_size][h_kv][d_h]: token t
 * of sequence b sits in page page_table[b * max_pages + t / page_size], row t % page_size.
 * p->k_strides / p->v_strides give the row (token) stride in [1] and the head stride in [2], in
 * elements ([0] is unused); k_page_stride / v_page_stride are the elements between consecutive
 * pages.  page_size must be a multiple of 64 and of the chunk B (a chunk never straddles two
 * pages), max_pages * page_size >= p->seqlen, and every page that holds a position < seqlen_b
 * (after the append) must be mapped.  bf16 with d_h = 128 only (other configurations return
 * DASH_EUNSUPPORTED).  The page table is read by the kernels on the device; it may change
 * between calls (the caller owns the allocation policy).  Results equal the contiguous-cache
 * calls bit for bit. */
typedef struct {
    const int* page_table;            /* device int32 [batch, max_pages] */
    int max_pages, page_size, num_pages;
    long long k_page_stride, v_page_stride;
} dash_paged_kv;

/* dash_summary_build / dash_summary_append / dash_decode on paged caches (same arguments plus
 * the page description; K_pool / V_pool take the place of K_cache / V_cache). */
int dash_summary_build_paged(const dash_params* p, const dash_paged_kv* pk, const void* K_pool,
                             const float* qbar, const int* seqlens, float* kbar_cache, float* partial_state,
                             void* stream);
int dash_summary_append_paged(const dash_params* p, const dash_paged_kv* pk, const void* k_new,
                              const void* v_new, const float* qbar, void* K_pool, void* V_pool,
                              float* kbar_cache, float* partial_state, int* seqlens, void* stream);
int dash_decode_paged(const dash_params* p, const dash_paged_kv* pk, const void* q, const void* K_pool,
                      const void* V_pool, const float* kbar_cache, const int* seqlens, void* O,
                      const dash_route_out* route, void* workspace, size_t ws_bytes, void* stream);

/* dash_decode without a workspace, for callers that cannot obtain device memory of their own
 * (for example a plugin inside a runtime that owns every device allocation and gives it no
 * allocator, or a service that must not grow its device footprint once running).  The paper has
 * no counterpart; this is a deployment variant of dash_decode with the same arguments minus
 * route/workspace, and the same results bit for bit.
 *   Scratch: a fixed 16 MiB device array inside the library (one per GPU that loads it, held
 *   until the process exits).  A request whose decode workspace, dash_workspace_size(p,
 *   DASH_OP_DECODE), exceeds 16 MiB returns DASH_EWORKSPACE before anything is enqueued; invalid
 *   parameters return what dash_decode would (DASH_EINVAL or DASH_EUNSUPPORTED).
 *   status: device int32 written on the stream after the decode kernels: 0, or the non-zero code
 *   of a bounded on-chip wait that timed out (the output is then not valid).  NULL skips it.
 *   The array is shared by every call on a GPU and keeps the last call's contents (each call
 *   writes every scratch value before reading it): calls whose kernels overlap on the GPU race
 *   and must be serialised by the caller.
 *   The array's device address is looked up the first time the call runs under a given (device,
 *   CUDA context) pair, with that device current, and cached for that pair; make that first call
 *   before any stream capture.
 *   Allocates nothing (no cudaMalloc / cudaFree / allocating library routine). */
int dash_decode_noalloc(const dash_params* p, const void* q, const void* K_cache, const void* V_cache,
                        const float* kbar_cache, const int* seqlens, void* O, int* status, void* stream);

/* Backward pass of dash_prefill: gradients of L = sum(dO * O) with respect to Q, K, V and qbar.
 * The paper review page (section 3, the text after Eq. 9) states that the output is
 * differentiable in q, k, v and the prior, the gradient reaching the Stage 1 entmax scores and
 * through them the Stage 0 summaries; its Stage 2 kernel row says the training backward reuses
 * the routed support (the entmax Jacobian is sparse).  The routed set is piecewise constant in
 * the inputs: no gradient flows through its choice.
 *   Inputs: Q, K, V, qbar, p and the route lists (counts, chunk_idx, bias: all three required)
 *   and kbar_out of the dash_prefill call whose output is being differentiated; dO with O's
 *   layout (p->o_strides, p->dtype).
 *   Outputs (fp32, contiguous, overwritten): dQ [batch, n, h_q, d_h], dK, dV [batch, n, h_kv, d_h],
 *   dqbar [h_kv, d_h] (summed over the batch).
 *   Workspace: dash_workspace_size(p, DASH_OP_BACKWARD) bytes (per-row log-sum-exp, the chunk
 *   logit gradients per routed entry, the route lists transposed per chunk), 256-byte aligned.
 *   DASH_EUNSUPPORTED when g_q * floor(n / B) chunk logits of one position do not fit the
 *   query-major kernel's shared memory (about 50K floats).  Deterministic: no atomics on
 *   floating-point results. */
int dash_backward(const dash_params* p, const void* Q, const void* K, const void* V, const float* qbar,
                  const void* dO, const float* kbar, const dash_route_out* route, float* dQ, float* dK, float* dV,
                  float* dqbar, void* workspace, size_t ws_bytes, void* stream);

/* Diagnostic knob: the number of polls after which a bounded on-chip wait of the tensor-core
 * Stage 2 prefill kernels gives up (the kernel then sets the workspace status word, drains its
 * in-flight copies and MMAs, frees its tensor memory and returns; the output is not valid).  It
 * applies to launches enqueued after the call; 0 makes the first wait give up at once (used by the
 * tests of that failure path).  The default is 2^23.  Returns the previous limit, or -1 for a
 * negative argument (nothing changed).  Not thread-safe with respect to concurrent launches. */
long long dash_set_wait_limit(long long polls);

/* Static text for a status code. */
const char* dash_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* DASH_H */
