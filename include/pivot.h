/*
 * pivot.h -- C ABI of the B200 (sm_100a) PIVOT query-group indexer.
 *
 * The operation is the indexer of token-level sparse attention and its PIVOT
 * replacement, as described in "PIVOT: Efficient Query-Group Indexing for
 * Token-Level Sparse Attention" (arXiv 2607.24593): the pages "PIVOT explained
 * -- from paper to working code in 10 minutes" (sections "The Problem", "How It
 * Works", "Show Me The Code") and the paper's abstract.
 *
 * Common conventions (all entry points):
 *  - Tensors are row-major, bfloat16 for q and k ("const void*" pointing to
 *    2-byte bf16 values), int32 for indices.  All tensor pointers are DEVICE
 *    pointers, 16-byte aligned.  The caller owns every buffer; the library keeps
 *    no pointer after the call returns.
 *  - Calls are asynchronous: work is enqueued on `stream` (a cudaStream_t passed
 *    as void*; NULL = the legacy default stream) and the call returns without
 *    synchronising.  Outputs are valid once the stream has reached that point.
 *  - Scores are unscaled dot products q . k.  A query at position pos may only
 *    select keys j < pos.  Ties in score go to the lower key index.  Every
 *    output row holds its selected key indices in ascending order, followed by
 *    -1 padding up to top_k.
 *  - head_dim d must be 64 or 128; 1 <= top_k <= Kc <= 4096.
 *  - Return value: PIVOT_OK, or an error code with a message available from
 *    pivot_last_error() (thread-local).  Argument errors are detected on the
 *    host before anything is enqueued.  Errors raised by the kernels (a bounded
 *    wait that gave up, an over-long decode sequence) are reported by
 *    pivot_sync_status().
 *  - There is no CPU fallback: on a machine without an sm_100 device every
 *    call returns PIVOT_ERR_UNSUPPORTED.
 */
#ifndef PIVOT_H_
#define PIVOT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PIVOT_REFINE = 0, PIVOT_REUSE = 1 } pivot_mode_t;

/*
 * Option bit OR-ed into `mode`: scan with the group mean rounded to bf16
 * instead of the fp32 mean.  This is a variant of the method, not the method:
 * the pages define the proxy as the group mean ("How It Works": proxy_q =
 * mean(group)) and this library takes it in fp32 by default, which the
 * tensor-core scan carries as three bf16 terms (three MMA passes per key
 * tile).  With the flag the scan makes one pass; candidate sets then differ
 * from the fp32-mean ones wherever the bf16 rounding reorders near-boundary
 * keys.
 */
enum { PIVOT_PROXY_BF16 = 0x100 };

/*
 * Option bit OR-ed into PIVOT_REFINE (prefill entry points only): the
 * listing's reading of Refine ("Show Me The Code", pivot_refine, which scans
 * k[:pos] for each member): member pos takes its candidate set from the group
 * proxy's scores over its own prefix j < pos, instead of one set per group
 * over j < last.  A fidelity variant, not the method's one shared scan: the
 * scan runs once per member (rows = positions) and every member gathers its
 * own candidates.  Its candidate rows hold L*H*ceil(Kc/128)*128 int32 of the
 * workspace; out_cand (when given) is then [L,H,Kc].  Decode entry points and
 * PIVOT_REUSE return PIVOT_ERR_INVALID_ARG with this bit.
 */
enum { PIVOT_PER_MEMBER_SCAN = 0x200 };

typedef enum {
  PIVOT_OK = 0,
  PIVOT_ERR_INVALID_ARG = 1,
  PIVOT_ERR_UNSUPPORTED = 2,
  PIVOT_ERR_CUDA = 3,
  PIVOT_ERR_TIMEOUT = 4,
  PIVOT_ERR_WORKSPACE = 5
} pivot_status_t;

/*
 * PIVOT prefill indexer for one layer, all heads.
 * Paper abstract and "How It Works": consecutive queries form groups of g
 * (starting at 0, g, 2g, ...; the last may be partial); each group's proxy is
 * the mean of its queries (fp64 sum divided by the member count, rounded to
 * fp32); one scan of the proxy over the group's causal prefix gives a
 * candidate set.
 *   mode = PIVOT_REFINE ("How It Works" per-query refine; listing pivot_refine):
 *     scan keys j < last (the group's largest position), C = top-min(Kc,last);
 *     member pos re-scores {j in C : j < pos} with its own query and keeps
 *     top-min(top_k, that count).
 *   mode = PIVOT_REUSE (listing pivot_reuse): scan keys j < s (group start);
 *     every member gets the proxy's top-min(top_k, s).  Kc is not used.
 *   Either may be OR-ed with PIVOT_PROXY_BF16 (the bf16-proxy variant);
 *   PIVOT_REFINE also with PIVOT_PER_MEMBER_SCAN (the listing's per-member
 *   scan).
 * q, k:     bf16 [L][H][d].
 * out_idx:  int32 [L][H][top_k].
 * Temporary device memory is taken with cudaMallocAsync on `stream` and freed
 * on it before return (see pivot_index_ws to supply it instead).
 */
int pivot_index(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                int32_t* out_idx, void* stream);

/*
 * Dense indexer -- the per-query scan that PIVOT replaces ("The Problem": every
 * query scores every preceding token and keeps the top-k).
 * out_idx[pos][h] = top-min(top_k, pos) of q[pos,h] . k[j,h] over j < pos.
 * q, k bf16 [L][H][d]; out_idx int32 [L][H][top_k].
 */
int dense_index(const void* q, const void* k, int L, int H, int d, int top_k, int32_t* out_idx,
                void* stream);

/*
 * PIVOT decode indexer for one multi-token-prediction step over a batch of
 * sequences (paper abstract: in decode a group is the queries decoded together
 * in one MTP step).  Sequence b holds n_b context keys plus the g keys of this
 * step in the packed cache rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 * (n_b = cu_seqlens[b+1] - cu_seqlens[b] - g >= 0); its g queries sit at
 * positions n_b .. n_b+g-1.  Refine scans j < n_b+g-1 and keeps top-min(Kc, .)
 * candidates; Reuse scans j < n_b.  Indices are positions within the sequence.
 * q:          bf16 [B][g][H][d].
 * kcache:     bf16 [cu_seqlens[B]][H][d].
 * cu_seqlens: int32 [B+1], device memory, non-decreasing.
 * max_seqlen: an upper bound on cu_seqlens[b+1]-cu_seqlens[b] for every b; a
 *             longer sequence is skipped on the device and reported by
 *             pivot_sync_status() as PIVOT_ERR_INVALID_ARG.
 * out_idx:    int32 [B][g][H][top_k].
 */
int pivot_decode_index(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d,
                       int g, int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx, void* stream);

/*
 * Workspace-taking variants: identical results; `workspace` (device, 256-byte
 * aligned, owned by the caller, contents ignored) must hold at least the
 * number of bytes reported by the matching *_workspace_size call, otherwise
 * PIVOT_ERR_WORKSPACE is returned and nothing runs.  out_scores (nullable,
 * float32, same shape as out_idx) receives the score that decided each output
 * index -- the member query's score for Refine and dense, the proxy's score
 * for Reuse -- and NaN in the padding.
 */
size_t pivot_workspace_size(int L, int H, int d, int g, int top_k, int Kc, int mode);
int pivot_index_ws(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                   int32_t* out_idx, float* out_scores, void* workspace, size_t workspace_bytes, void* stream);

size_t dense_workspace_size(int L, int H, int d, int top_k);
int dense_index_ws(const void* q, const void* k, int L, int H, int d, int top_k, int32_t* out_idx,
                   float* out_scores, void* workspace, size_t workspace_bytes, void* stream);

size_t pivot_decode_workspace_size(int B, int H, int d, int g, int top_k, int Kc, int mode, int max_seqlen);
int pivot_decode_index_ws(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d,
                          int g, int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx,
                          float* out_scores, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The sparse attention that consumes the index rows ("Show Me The Code": the
 * demo after pivot_refine): for query row r, head h and the valid entries J of
 * idx[r][h] (>= 0; -1 is padding),
 *     out[r][h] = sum_{j in J} softmax_j((q[r][h] . k_j) * d^-1/2) v_j,
 * with fp32 arithmetic; a row without a valid index gets zeros.
 *   q:   bf16 [R][H][d]; prefill R = L, decode R = B*g (q of pivot_decode_index).
 *   k,v: bf16; prefill [L][H][d] (index j = key row j); decode the packed cache
 *        [rows][H][d] with cu_seqlens (device [B+1], index j of sequence
 *        r / g = cache row cu_seqlens[r / g] + j); cu_seqlens NULL = prefill.
 *   idx: int32 [R][H][top_k] (the indexer's output rows); every valid index
 *        must address a key of its sequence -- it is not checked.
 *   out: float32 [R][H][d].
 * Asynchronous on `stream`; no workspace.  Returns PIVOT_OK,
 * PIVOT_ERR_INVALID_ARG or PIVOT_ERR_UNSUPPORTED (d not 64/128, no sm_100).
 */
int pivot_sparse_attention(const void* q, const void* k, const void* v, const int32_t* idx,
                           const int32_t* cu_seqlens, int R, int H, int d, int g, int top_k, float* out,
                           void* stream);

/*
 * MTP decode over a paged key cache (the layout of paged-attention serving
 * engines).  kpages: bf16 [num_pages][page_size][H][d].  block_table: int32
 * [B][max_pages] (device) maps sequence b's logical page p -- its keys
 * p*page_size .. p*page_size + page_size - 1 -- to a page of kpages.
 * seqlens: int32 [B] (device), the cache rows n_b + g that sequence b holds.
 * page_size must be a power of two and max_pages * page_size >= max_seqlen
 * (else PIVOT_ERR_INVALID_ARG).  Every page id that a sequence's first
 * seqlens[b] keys use must index a page of kpages: the tables live on the
 * device and are not checked.  Everything else -- q, the outputs, the
 * workspace (pivot_decode_workspace_size), sequences longer than max_seqlen
 * -- is as in pivot_decode_index_ws, and the results equal those of the same
 * sequences packed contiguously.
 */
int pivot_decode_index_paged(const void* q, const void* kpages, const int32_t* block_table, const int32_t* seqlens,
                             int B, int H, int d, int g, int page_size, int max_pages, int top_k, int Kc, int mode,
                             int max_seqlen, int32_t* out_idx, float* out_scores, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * As the _ws variants, with two more nullable outputs that expose the
 * method's intermediate results ("How It Works": the proxy of each group and
 * its candidate set C = top-Kc of the proxy scores):
 *   out_proxy: float32 [G][H][d] (decode: [B][H][d]), each group's proxy --
 *              the fp32 mean of its queries (or its bf16 rounding under
 *              PIVOT_PROXY_BF16), 16-byte aligned;
 *   out_cand:  int32 [G][H][Kc] (decode: [B][H][Kc]), PIVOT_REFINE only (else
 *              PIVOT_ERR_INVALID_ARG): each group's candidate key indices in
 *              ascending order, -1 padded; a decode sequence skipped for its
 *              length gets an all -1 row.
 * G = ceil(L / g).
 */
int pivot_index_ex(const void* q, const void* k, int L, int H, int d, int g, int top_k, int Kc, int mode,
                   int32_t* out_idx, float* out_scores, float* out_proxy, int32_t* out_cand, void* workspace,
                   size_t workspace_bytes, void* stream);
int pivot_decode_index_ex(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d, int g,
                          int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx, float* out_scores,
                          float* out_proxy, int32_t* out_cand, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Decode without any device allocation (the paper has no counterpart; this is
 * a deployment variant of pivot_decode_index, same arguments and results).
 * For callers that cannot allocate device memory during a decode step: an
 * inference engine that has already handed all free HBM to its KV-cache pool,
 * so a cudaMalloc there would fail or fragment it, or host code that has no
 * allocator of its own and must not own device buffers.  Its scratch is a
 * 32 MiB array built into the library (held by every GPU that loads it until
 * the process exits); a call whose scratch need -- proxies B*H*d*4 + order keys
 * H*B*max_seqlen*4 + (Refine) candidates H*B*CW*4 bytes, CW = Kc rounded up to
 * a multiple of 128, each rounded up to 256 -- exceeds 32 MiB is rejected with
 * PIVOT_ERR_WORKSPACE and a message.
 * The first call on each device looks the array's address up (once, with that
 * device current); make that first call before any stream capture.  All calls
 * share the one array and it keeps the previous call's contents (nothing in it
 * needs to start at zero): calls that may overlap on the GPU -- concurrent
 * streams, or several host threads -- race on it and must be serialised by the
 * caller.
 */
int pivot_decode_index_noalloc(const void* q, const void* kcache, const int32_t* cu_seqlens, int B, int H, int d,
                               int g, int top_k, int Kc, int mode, int max_seqlen, int32_t* out_idx,
                               float* out_scores, void* stream);

/*
 * Synchronises `stream`, then reads and clears this device's kernel status
 * word.  Returns PIVOT_OK, PIVOT_ERR_TIMEOUT (a bounded wait inside a kernel
 * gave up; that call's outputs are not valid), PIVOT_ERR_INVALID_ARG (a decode
 * sequence exceeded max_seqlen) or PIVOT_ERR_CUDA (a CUDA error, or status bit
 * 8: a refine selection exceeded its round limit, which finite scores never
 * do; that call's outputs are not valid).  *flags (nullable) receives the raw
 * status bits; bit 4 means some rows took the exact fallback path (results
 * remain exact).
 */
int pivot_sync_status(void* stream, int* flags);

/*
 * Launch trace (profiling aid, off by default; per calling thread).  While
 * enabled, every kernel launch of this library is bracketed by two CUDA events
 * recorded on the launch stream.  pivot_trace_collect() waits for the recorded
 * events, aggregates them by kernel name and clears the trace: names receives a
 * comma-separated list, ms[i] the summed device time of kernel i, count[i] its
 * launches (up to max_items kernels).  Returns the number of kernels, or a
 * negated error code.
 */
int pivot_trace_enable(int on);
int pivot_trace_collect(char* names, size_t names_len, float* ms, int* count, int max_items);

/*
 * Testing aid (the method has no counterpart).  Every wait of a kernel on
 * another of its roles (an mbarrier phase) gives up after a limit, raises the
 * status that pivot_sync_status() reports as PIVOT_ERR_TIMEOUT, drains what it
 * had issued and returns; no kernel traps or spins for ever.  This sets that
 * limit, in nanoseconds, for the calls that follow in this process (0 restores
 * the default of 2 seconds).  A tiny limit makes a call time out on purpose;
 * its outputs are then not valid.  Returns PIVOT_OK.
 */
int pivot_set_wait_limit(unsigned long long ns);

/* Message of the last error on the calling thread ("" if none). */
const char* pivot_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PIVOT_H_ */
