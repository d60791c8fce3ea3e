/*
 * saf3r.h - C ABI of the head-wise dynamic sparse global attention library.
 *
 * The method is SAF3R ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D
 * Reconstruction Transformers", arXiv 2607.03612).  Every attention head of a
 * cross-view global-attention layer gets its own key/value index set, chosen
 * by one of four kernels (section 4.1): a static position/anchor pattern, a
 * mean-query-probe Top-K (vertical-line heads), a DINO-feature Top-K
 * (correspondence heads) or a uniform stride (scanning heads).  Exact softmax
 * attention then runs over the kept keys only; the dynamic sets are built once
 * per input and cached (section 4.3); an offline step picks each head's
 * configuration from the output NMSE against full attention (section 4.2).
 *
 * Conventions shared by every call
 *   - Token layout: S views; each view holds n_special special tokens
 *     (camera, registers) followed by grid_h*grid_w patch tokens in raster
 *     order.  V = n_special + grid_h*grid_w, N = S*V, token t = s*V + i.
 *   - Q, K, V, O are row-major [H][N][d] tensors (bf16 inputs; bf16 or fp32
 *     output), d = 64, rows of 128 bytes.  DINO features are fp32
 *     [S*grid_h*grid_w][dino_dim], one row per patch token in token order.
 *   - All pointers named q, k, v, dino, out, cache and workspace are DEVICE
 *     pointers, 16-byte aligned.  `stream` is a cudaStream_t (NULL = legacy
 *     default stream).  The caller owns every buffer; the library allocates
 *     no device memory and keeps no state except one error word per device.
 *   - Calls are asynchronous on `stream` unless stated.  Argument errors are
 *     returned at once and launch nothing.  Errors found on the device (a
 *     bounded wait that expired, an index cache built for another layout)
 *     are recorded in the device error word and reported by saf3r_check().
 *   - Attention scale is 1/sqrt(d); excluded keys take no part in the softmax
 *     (their logit is -inf), so each row is an exact softmax over its kept set.
 */
#ifndef SAF3R_H
#define SAF3R_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAF3R_OK = 0,
    SAF3R_ERR_INVALID = 1,      /* bad argument, or cache/layout mismatch found on the device */
    SAF3R_ERR_CUDA = 2,         /* a CUDA runtime/driver call failed */
    SAF3R_ERR_TIMEOUT = 3,      /* a bounded device wait expired; the kernel gave up cleanly */
    SAF3R_ERR_INDEX = 4,        /* an index read from the cache was out of range */
    SAF3R_ERR_UNSUPPORTED = 5   /* shape or device not supported (d != 64, not sm_100) */
} saf3r_status;

/* Head kinds (section 3, Observation #2; kernels of section 4.1). */
typedef enum {
    SAF3R_POSITION = 0,  /* static kernel: specials + anchor view 0 + the 3x3 cell neighbourhood in every view */
    SAF3R_PROBE = 1,     /* query-probe Top-K: Top-k patch keys by mean-query score, + all specials */
    SAF3R_CORR = 2,      /* DINO Top-K, block-wise: per 64-query tile, Top-k 64-token key tiles + all specials */
    SAF3R_SCAN = 3,      /* uniform sampling: keys j with j mod stride == phase, + all specials */
    SAF3R_DENSE = 4,     /* every key (full attention) */
    SAF3R_HYBRID = 5,    /* CORR's k key tiles united with SCAN's lattice (stride, phase), + all specials:
                            the Top-K / uniform-stride combination that section 5.3 ("Further Analysis
                            of the DINO Top-K kernel") proposes against regions the DINO matches miss */
    SAF3R_TOKEN = 6      /* DINO Top-K, token-wise: a patch query keeps, in every frame, the k patch tokens of
                            highest DINO cosine (section 4.1; section 5.1 sets k per frame), + all specials;
                            a special-token query (no DINO feature) keeps every key */
} saf3r_head_type;

typedef struct {
    int32_t S;          /* views, >= 1 */
    int32_t grid_h;     /* patch rows per view */
    int32_t grid_w;     /* patch columns per view */
    int32_t n_special;  /* special tokens per view (5: 1 camera + 4 registers) */
    int32_t H;          /* heads, 1..64 */
    int32_t d;          /* head dimension; must be 64 */
    int32_t dino_dim;   /* DINO feature width (384); 1..1024 */
    int32_t tile;       /* token tile of the block-wise DINO kernel; must be 64 */
} saf3r_layout;

typedef struct {
    int32_t type;       /* saf3r_head_type */
    int32_t k;          /* PROBE: kept patch keys (1..S*grid_h*grid_w); CORR, HYBRID: kept key tiles (1..T);
                           TOKEN: kept patch tokens per frame (1..grid_h*grid_w) */
    int32_t stride;     /* SCAN, HYBRID: >= 1 */
    int32_t phase;      /* SCAN, HYBRID: 0 <= phase < stride */
    int32_t radius;     /* POSITION: neighbourhood radius in cells, 0..3 (1 = 3x3); -1 = the anchor frame
                           only (section 4.1's first static example: all queries attend to view 0) */
} saf3r_head_cfg;

/* Operations for saf3r_workspace_bytes. */
enum { SAF3R_OP_SELECT = 0, SAF3R_OP_SPARSE = 1, SAF3R_OP_DENSE = 2, SAF3R_OP_PROFILE = 3 };

/*
 * Size in bytes of the index cache that saf3r_select_kv fills for this layout
 * and per-head configuration (cfg: H entries).  The cache holds a header with
 * a hash of (layout, cfg), each probe head's kept patch keys (int32, ascending)
 * and, if any head is CORR or HYBRID, the ranked key-tile list of every query
 * tile (int32 [T][kmax], best first; T = ceil(N/64), kmax = largest such k),
 * and, if any head is TOKEN, the ranked per-frame lists of every patch query
 * (int32 [S*P][S][kmax] patch indices, best first; kmax = largest TOKEN k),
 * and, where the layout allows (S*P patches, P up to about 6,000, at most
 * 2^28 union entries per budget), the patch queries' order for the tensor
 * cores plus, per distinct TOKEN k and per 256 queries of that order, room
 * for the union of their kept tokens (S * min(256 k, P) entries, int32) and
 * one 64-bit mask per query and 64 union entries: about
 * 36 * ceil(S*P/256) * S * min(256 k, P) bytes per distinct k (2.6 GB at
 * S = 100, P = 1369, k = 16).
 * Returns 0 for an invalid layout or cfg.
 */
size_t saf3r_cache_bytes(const saf3r_layout* layout, const saf3r_head_cfg* cfg);

/*
 * Size in bytes of the device workspace that operation `op` needs:
 * SAF3R_OP_SELECT or SAF3R_OP_SPARSE with the per-head cfg (H entries),
 * SAF3R_OP_DENSE with cfg = NULL.  Profiling uses
 * saf3r_profile_workspace_bytes.  Returns 0 for invalid arguments.
 */
size_t saf3r_workspace_bytes(const saf3r_layout* layout, const saf3r_head_cfg* cfg, int op);

/* Workspace bytes of saf3r_profile_heads for n_cand candidates. */
size_t saf3r_profile_workspace_bytes(const saf3r_layout* layout, const saf3r_head_cfg* cand, int n_cand);

/*
 * Build the per-input dynamic index sets (section 4.3, "Online Pattern
 * Adaptation") and write them to `cache` (saf3r_cache_bytes bytes).
 *   - PROBE heads: qbar = mean of all N query rows of the head (fp64 sum,
 *     rounded once to fp32); score_j = qbar . k_j / sqrt(d) in fp32; the k
 *     patch keys of highest score (ties to the lower token index) are kept.
 *     Section 4.3 shows this ranking equals ranking keys by the column means
 *     of Q K^T / sqrt(d).
 *   - CORR heads: each flat 64-token tile gets the mean of the L2-normalised
 *     DINO features of its patch tokens; tiles are compared by cosine; every
 *     query tile ranks all tiles (itself included; ties to the lower tile).
 *     Computed once and shared by all CORR and HYBRID heads (prefixes serve
 *     smaller k).
 *   - TOKEN heads: L2-normalised DINO features; for every patch query and
 *     every frame, the frame's patch tokens ranked by cosine (own token
 *     included; ties to the lower patch index); the lists are cached.
 *     The cosines are formed on the tensor cores (fp16 features, fp32
 *     accumulation, fp16 scores: within 2e-3 of the exact cosine) and every
 *     candidate within twice that bound of the k-th score is recomputed
 *     exactly (fp64), so the ranking is that of the fp64 cosines rounded to
 *     fp32.  The workspace then holds the fp16 scores of up to 1 GiB of query
 *     rows at a time.  Needs dino_dim <= 384 (SAF3R_ERR_UNSUPPORTED otherwise).
 *     The patch queries are then ordered by their best match in frame 0,
 *     then in frame 1 (queries that see the same scene point become
 *     neighbours), and every 256 queries of that order get the ascending
 *     union of their kept tokens and a per-query bitmask over it, which the
 *     attention streams through the tensor cores.
 *   - POSITION, SCAN and DENSE heads need no cached state (a HYBRID head's
 *     lattice neither).
 * q, k: bf16 [H][N][d]; dino: fp32 patch features, or NULL when no head is
 * CORR, HYBRID or TOKEN.
 * workspace: saf3r_workspace_bytes(layout, cfg, SAF3R_OP_SELECT) bytes.
 */
saf3r_status saf3r_select_kv(const saf3r_layout* layout, const saf3r_head_cfg* cfg,
                             const void* q, const void* k, const float* dino,
                             void* cache, void* workspace, void* stream);

/*
 * saf3r_select_kv without a caller workspace.  No counterpart in the paper: this
 * entry point exists for callers that cannot allocate device memory for the
 * workspace - engines whose latency-critical loop must not enter an allocator,
 * plug-in hosts that pass a library only its inputs and outputs.  It builds
 * exactly the cache saf3r_select_kv builds, taking its scratch from a 40 MiB
 * device array compiled into the library (held by every GPU that loads the
 * library until the process exits), and calls no allocator.
 *   - Limit: saf3r_workspace_bytes(layout, cfg, SAF3R_OP_SELECT) must be at most
 *     40 MiB (41943040 bytes; the 274,800-token layer with 4 probe and 4
 *     correspondence heads needs 32.3 MiB); larger layers return
 *     SAF3R_ERR_UNSUPPORTED and launch nothing.
 *   - First-call setup: the first call on each device looks up the array's
 *     device address (cudaGetSymbolAddress) and remembers it; later calls on
 *     that device reuse it.
 *   - All calls share the one array: calls that may overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the caller.
 *     Nothing in the array needs to start at zero; each call clears what it needs.
 * Arguments and errors as saf3r_select_kv.
 */
saf3r_status saf3r_select_kv_static(const saf3r_layout* layout, const saf3r_head_cfg* cfg,
                                    const void* q, const void* k, const float* dino,
                                    void* cache, void* stream);

/*
 * Sparse global attention over cached index sets (section 4.1): for every head
 * h and query i, O[h][i] = sum_{j in kept(h,i)} softmax_j(q.k_j/sqrt(d)) v_j.
 * `cache` must come from saf3r_select_kv with the same layout and cfg (checked
 * on the device through the cache header hash; a mismatch records
 * SAF3R_ERR_INVALID and leaves `out` unwritten).  q, k, v may be fresh
 * tensors of a later layer call: the cached sets are reused as they are.
 * All heads run in one tensor-core launch; a TOKEN head's patch queries run
 * there over their cached per-256-query key unions (each query masked to its
 * own keys) when the layout has unions and the launch's per-head plans fit
 * (at most 64 plans: one per head, plus one per TOKEN head with special
 * tokens), else in a per-query gather kernel.  Both give the exact softmax
 * over each query's kept keys.
 * out: bf16 [H][N][d] (out_is_fp32 = 0) or fp32 (out_is_fp32 = 1).
 * workspace: saf3r_workspace_bytes(layout, cfg, SAF3R_OP_SPARSE) bytes.
 */
saf3r_status saf3r_sparse_attn(const saf3r_layout* layout, const saf3r_head_cfg* cfg, const void* cache,
                               const void* q, const void* k, const void* v,
                               void* out, int out_is_fp32, void* workspace, void* stream);

/*
 * Full attention over all N keys for every head: O_full of section 4.2, the
 * reference of the per-head NMSE.  Layout arguments as saf3r_sparse_attn.
 * workspace: saf3r_workspace_bytes(layout, NULL, SAF3R_OP_DENSE) bytes.
 */
saf3r_status saf3r_dense_attn(const saf3r_layout* layout, const void* q, const void* k, const void* v,
                              void* out, int out_is_fp32, void* workspace, void* stream);

/*
 * Offline head profiling (section 4.2) on one calibration input.  For every
 * candidate c (n_cand entries; a SCAN candidate's phase is replaced by
 * head mod stride) and every head h it computes
 *     nmse[h*n_cand + c]  = ||O_full - O_c||^2 / ||O_full||^2        (eq. 1)
 *     pairs[h*n_cand + c] = number of (query, kept key) pairs (Omega = 4*d*pairs)
 * and chooses for each head the candidate of least Omega whose NMSE is at
 * most nmse_max (ties to the lower candidate index); when none qualifies, the
 * candidate of least NMSE (the argmin of eq. 2).  chosen (H entries), nmse
 * and pairs are HOST arrays.  Synchronizes `stream`.
 * workspace: saf3r_profile_workspace_bytes(layout, cand, n_cand) bytes.
 */
saf3r_status saf3r_profile_heads(const saf3r_layout* layout, const saf3r_head_cfg* cand, int n_cand,
                                 const void* q, const void* k, const void* v, const float* dino,
                                 double nmse_max, saf3r_head_cfg* chosen, double* nmse, int64_t* pairs,
                                 void* workspace, void* stream);

/*
 * The search of section 4.2, eq. 2 ("progressive local substitution"), as a
 * host-side rule over the tables saf3r_profile_heads measured on each input
 * of a calibration set.  Per head h and candidate c it averages eq. 1 over
 * the n_inputs inputs (E[h][c], fp64 sum in input order / n_inputs) and the
 * kept pairs likewise (W[h][c], the cost: Omega = 4*d*pairs, so comparisons of
 * pairs are comparisons of Omega).  Then, per head, it starts from the
 * baseline candidate `base` (the uniform-stride SCAN candidate at the target
 * sparsity sigma: stride ceil(1 / (1 - sigma))) and visits the other
 * candidates in index order, making c the current choice when
 * W[h][c] <= W[h][base] and E[h][c] < E[h][current].  The result minimises the
 * error under the baseline's cost; ties go to the baseline, then to the lower
 * candidate index.
 *
 * nmse:  HOST double  [n_inputs][H][n_cand] (saf3r_profile_heads' nmse, per input)
 * pairs: HOST int64   [n_inputs][H][n_cand] (saf3r_profile_heads' pairs, per input)
 * choice: HOST int32  [H] out, the chosen candidate index per head
 * nmse_mean: HOST double [H][n_cand] out (E), or NULL
 * Returns SAF3R_ERR_INVALID for null inputs, n_inputs, H or n_cand < 1, or
 * base out of range.  No device work, no stream.
 */
saf3r_status saf3r_choose_eq2(int n_inputs, int H, int n_cand, const double* nmse, const int64_t* pairs,
                              int base, int32_t* choice, double* nmse_mean);

/*
 * Stride of the uniform-sampling baseline from which the eq. 2 search starts
 * (section 4.2: uniform sampling at sparsity ratio sigma; section 5.1 uses
 * sigma = 0.85): keeping one key in s has sparsity 1 - 1/s, so the baseline
 * stride is the smallest s with 1 - 1/s >= sigma, i.e. ceil(1 / (1 - sigma))
 * (7 for sigma = 0.85).  Returns -1 for sigma outside [0, 1).  Host only.
 */
int32_t saf3r_baseline_stride(double sigma);

/*
 * Copy one head's cached index list to host memory (synchronizes `stream`):
 * PROBE head -> its k kept patch keys (ascending); CORR or HYBRID head -> the
 * ranked tile list int32 [T][k] truncated to that head's k; TOKEN head -> the
 * per-frame lists int32 [S*P][S][k] (patch indices) truncated to its k.  *n receives the number
 * of entries; at most `cap` are written.  Other head kinds return
 * SAF3R_ERR_INVALID.
 */
saf3r_status saf3r_cache_export(const saf3r_layout* layout, const saf3r_head_cfg* cfg, const void* cache,
                                int head, int32_t* host_idx, size_t cap, size_t* n, void* stream);

/*
 * Exact number of (query, kept key) pairs of every head under (layout, cfg)
 * with the index sets held in `cache` (section 4.2: the cost of a
 * configuration is Omega = 4*d*pairs FLOPs).  pairs: HOST int64 [H].
 * Synchronizes `stream` (the correspondence heads' tile lists are read back).
 */
saf3r_status saf3r_kept_pairs(const saf3r_layout* layout, const saf3r_head_cfg* cfg, const void* cache,
                              int64_t* pairs, void* stream);

/*
 * Timing hook for measurement: when start and stop are both non-NULL
 * cudaEvent_t handles, every following saf3r_sparse_attn / saf3r_dense_attn
 * call made on this host thread records `start` on its stream right before
 * its attention kernel and `stop` right after it.  NULL, NULL switches the
 * hook off.  The events are owned by the caller.
 */
void saf3r_set_kernel_events(void* start, void* stop);

/*
 * Budget, in GPU clock cycles, of every bounded device wait (the attention
 * kernel's and the token-wise selection's pipeline waits) in the calls that
 * follow on this host thread; cycles <= 0 restores the default of 4e9 cycles
 * (about 2 s at 1.965 GHz).  When a wait runs out, its CTA records
 * SAF3R_ERR_TIMEOUT in the device error word, lets the copies it has in flight
 * land (a separate, fixed teardown budget), frees its tensor memory and exits;
 * the output rows of its unfinished work items are then left unwritten.
 */
void saf3r_set_wait_budget(long long cycles);

/*
 * Test hook for the timeout path.  The next saf3r_sparse_attn or
 * saf3r_dense_attn call on this host thread launches its attention kernel with
 * one softmax warp of the first CTA withholding its first "P is in tensor
 * memory" arrival, so the tensor-core warp's wait for it runs out after the wait
 * budget (see saf3r_set_wait_budget): nothing faults or hangs, every device wait
 * being bounded.  saf3r_check then returns SAF3R_ERR_TIMEOUT; the following
 * calls run normally.  Not for production use.
 */
void saf3r_test_withhold_arrive(void);

/*
 * Synchronize `stream`, then read and clear the calling device's error word.
 * Returns SAF3R_OK or the first device-side error recorded since the last check.
 */
saf3r_status saf3r_check(void* stream);

/* Number of kernels the last saf3r_* call on this host thread launched. */
int saf3r_last_launch_count(void);

/* Static text for a status code. */
const char* saf3r_status_string(saf3r_status status);

#ifdef __cplusplus
}
#endif

#endif /* SAF3R_H */
