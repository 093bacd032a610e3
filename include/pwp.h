/*
 * pwp.h -- C ABI of the B200 layer-reconstruction pruning library (libpwp.so).
 *
 * One linear layer W (c x b, rows = outputs, columns = input features) and its
 * calibration activations X (the pages' X is b x n with examples as columns; it
 * is passed here token-major, [n, b], the PyTorch activation layout) are turned
 * into a pruned and reconstructed W-hat and a pruning mask, following
 *   "Pruning LLMs with Thanos" (sections "The layer-reconstruction lens",
 *   "Contribution one: solve a selected set directly", "Contribution two: keep
 *   the budget global and the execution local") and, for the column-sequential
 *   special case, "Weight Pruning in Large Language Models ..." (llms.blog),
 *   section "SparseGPT: Second-Order Reconstruction at Scale".  The same page's
 *   sections "Wanda: Pruning by Weights and Activations", "The Failure of Magnitude
 *   Pruning in Large Transformers" and "N:M Semi-Structured Sparsity (2:4 Pattern)"
 *   define the no-update methods (PWP_WANDA, PWP_MAGNITUDE) and the compressed 2:4
 *   storage (pwp_pack_24).
 *
 * Conventions for every entry point:
 *   - All pointers named *_dev are device pointers; the caller owns every buffer.
 *     The library allocates no device memory: all scratch comes from the caller's
 *     workspace `ws` of `ws_bytes` bytes (at least 256-byte aligned), or, for
 *     pwp_prune_layer_noalloc, from one static array inside the library.  A call may
 *     create CUDA streams and events of its own and release them before it returns:
 *     the factor puts its next diagonal block on a side stream (three events; not
 *     while `stream` is being captured into a graph), the host entry points put their
 *     copies on copy streams; `stream` waits for all of that work, so it stays ordered
 *     as if it had been enqueued on `stream` itself.  The optional event timing
 *     (pwp_profile_enable) keeps its events until it is switched off.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and the call returns without synchronising.
 *   - Argument errors are detected on the host before anything is enqueued and
 *     returned synchronously (PWP_EINVAL, PWP_EWORKSPACE).  A CUDA launch error
 *     returns PWP_ECUDA.
 *   - Errors found on the device (a non-positive pivot, a wait that ran out, an
 *     unreachable budget) are written to the caller's device-resident pwp_stats
 *     (`status`, `status_site`); every later kernel of the same call becomes a
 *     no-op.  The caller reads `stats_dev` after synchronising the stream.
 *   - Calls on different streams with different workspaces are independent;
 *     two calls that share a workspace must be ordered by the caller.
 */
#ifndef PWP_H
#define PWP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PWP_OK = 0,
    PWP_EINVAL = 1,      /* bad shape, pattern, sparsity, block or dtype */
    PWP_ENOTSPD = 2,     /* damped Hessian not positive definite (pivot <= 0) */
    PWP_EWORKSPACE = 3,  /* workspace missing, misaligned or too small */
    PWP_ECUDA = 4,       /* a CUDA launch or runtime call failed */
    PWP_ETIMEOUT = 5,    /* a bounded device-side wait gave up */
    PWP_EBUDGET = 6      /* the unstructured target could not be reached */
} pwp_status;

typedef enum { PWP_THANOS = 0, PWP_SPARSEGPT = 1, PWP_WANDA = 2, PWP_MAGNITUDE = 3 } pwp_method;
typedef enum { PWP_UNSTRUCTURED = 0, PWP_NM = 1 } pwp_pattern;
typedef enum { PWP_BF16 = 0, PWP_FP32 = 1 } pwp_dtype;

/* Method configuration ("Thanos - Method of Pruning LLMs", section "Usage":
 * --prune_method, --sparsity_ratio, --sparsity_type).
 *   method   : PWP_THANOS (joint row solves, dynamic global budget) or
 *              PWP_SPARSEGPT (column-sequential OBS, per-block quota), or one of the
 *              no-update baselines of the llms.blog page: PWP_WANDA (score
 *              |W_kq| * ||X_q||, section "Wanda: Pruning by Weights and Activations")
 *              and PWP_MAGNITUDE (score |W_kq|, section "The Failure of Magnitude
 *              Pruning in Large Transformers"); both remove floor(sparsity * b) weights
 *              of every row (ties: lower column first), or the nm_m - nm_n lowest of
 *              every group, and change no other weight; block and damp are ignored.
 *   pattern  : PWP_UNSTRUCTURED, or PWP_NM with 0 < nm_n < nm_m <= 32 (keep nm_n of
 *              every nm_m consecutive weights of a row; groups start at column 0).
 *   sparsity : fraction of weights removed, 0 <= sparsity < 1 (ignored for PWP_NM).
 *   block    : column block width B, 1 <= B <= 128; for PWP_NM a multiple of nm_m
 *              (Thanos and SparseGPT only).
 *   damp     : lambda = damp * mean(diag H) of the undamped H, damp >= 0.
 *   alpha    : fraction of rows kept dense as outliers, 0 <= alpha < 1 (Thanos and
 *              SparseGPT; 0 for the others).  "Pruning LLMs with Thanos", section
 *              "Thanos versus SparseGPT on LLaMA-3 8B": alpha = 0.1 keeps 10% of the rows,
 *              so 2:4 and 4:8 prune 45% of the layer instead of 50%.  The page does not say
 *              which rows; here the floor(alpha * c) rows with the largest
 *              sum_q W_kq^2 ||X_q||^2 (ties: lower row first) are returned unchanged (mask 0)
 *              and the other rows are pruned as a layer of their own with this
 *              configuration (the unstructured budget is floor(sparsity * rows * b) of their
 *              weights). */
typedef struct {
    int32_t method;
    int32_t pattern;
    int32_t nm_n;
    int32_t nm_m;
    float sparsity;
    int32_t block;
    float damp;
    float alpha;
} pwp_config;

/* Device-resident results of one prune call (the caller allocates it in device
 * memory and reads it back after the stream is synchronised). */
typedef struct {
    int32_t status;          /* pwp_status found on the device, PWP_OK otherwise */
    int32_t status_site;     /* index of the kernel that first set `status` */
    int64_t pruned;          /* number of mask entries set (weights removed) */
    int64_t target;          /* floor(sparsity*c*b) for Thanos unstructured, else the
                                number of removals the pattern implies */
    float lambda;            /* damping actually added to the diagonal */
    int32_t shortfall;       /* 1 if a block wanted more removals than it had weights */
    int32_t reread_blocks;   /* blocks whose exact threshold needed a second pass */
    int32_t tie_blocks;      /* blocks whose threshold fell on tied scores */
    int32_t reserved[4];
} pwp_stats;

/* Bytes of workspace pwp_prune_layer / pwp_prune_layer_x need for this
 * configuration and shape.  Returns 0 for an invalid configuration. */
size_t pwp_workspace_bytes(const pwp_config* cfg, int32_t c, int32_t b);

/* Hessian accumulation, H (b x b fp32, row-major, full symmetric) :=
 *   beta * H + 2 X X^T     (pages' X = b x n; here X_dev is [n, b] token-major),
 * "Weight Pruning in Large Language Models ...", section "SparseGPT: Second-Order
 * Reconstruction at Scale" (H = 2 X X^T; damping is added later by the prune call).
 * Calling it repeatedly with beta = 1 streams calibration batches into one H.
 *   X_dev   : [n, b] elements of type xtype (PWP_BF16 or PWP_FP32), row stride b.
 *   n >= 0, 1 <= b <= 16384, beta in {0, 1}.  H_dev: b*b floats.
 * Needs no workspace. */
pwp_status pwp_hessian_accumulate(const void* X_dev, int32_t xtype, int64_t n, int32_t b,
                                  float* H_dev, int32_t beta, void* stream);

/* Damping and factorisation (the "Cholesky decomposition of H^-1 once per layer"
 * of the llms.blog SparseGPT section).  On entry H_dev holds the undamped
 * H = 2XX^T (b x b, row-major; only the upper triangle is read).  On return the
 * upper triangle of H_dev holds U, upper triangular with (H + lambda I)^-1 = U^T U,
 * lambda = damp * mean(diag H); the strict lower triangle is left unspecified.
 * g_diag_dev (b floats) receives diag(H)/2 = ||X_q||^2 before damping.
 * ws/ws_bytes: scratch of at least pwp_factor_workspace_bytes(b) bytes.
 * stats_dev receives lambda and a PWP_ENOTSPD status on a non-positive pivot. */
size_t pwp_factor_workspace_bytes(int32_t b);
pwp_status pwp_damp_factor(float* H_dev, int32_t b, float damp, float* g_diag_dev,
                           void* ws, size_t ws_bytes, pwp_stats* stats_dev, void* stream);

/* Prune one layer given its undamped Hessian.
 *   W_dev     : c x b row-major weights of type wtype (read only).
 *   H_dev     : undamped H = 2 X X^T (b x b fp32); DESTROYED (holds U on return) by
 *               PWP_THANOS and PWP_SPARSEGPT; PWP_WANDA reads only its diagonal
 *               (||X_q||^2 = H_qq / 2) and leaves it unchanged; PWP_MAGNITUDE does not
 *               use it (it may be NULL).
 *   W_out_dev : c x b fp32, receives W-hat (pruned entries exactly 0.0f).
 *   mask_dev  : c x b bytes, receives 1 where a weight was removed, else 0.
 *   1 <= c, 1 <= b <= 16384, c*b < 2^31.
 * Method: "Pruning LLMs with Thanos", sections "Contribution one" and
 * "Contribution two" (PWP_THANOS); llms.blog SparseGPT section (PWP_SPARSEGPT). */
pwp_status pwp_prune_layer(const pwp_config* cfg, const void* W_dev, int32_t wtype,
                           int32_t c, int32_t b, float* H_dev, float* W_out_dev,
                           uint8_t* mask_dev, void* ws, size_t ws_bytes,
                           pwp_stats* stats_dev, void* stream);

/* Same as pwp_prune_layer, but first builds H = 2 X X^T into H_dev (b x b fp32,
 * caller-owned scratch, overwritten) from token-major activations X_dev ([n, b]).
 * PWP_WANDA takes ||X_q|| straight from X (fp64 sums) and PWP_MAGNITUDE ignores X; for
 * these two H_dev is not used and may be NULL. */
pwp_status pwp_prune_layer_x(const pwp_config* cfg, const void* W_dev, int32_t wtype,
                             int32_t c, int32_t b, const void* X_dev, int32_t xtype,
                             int64_t n, float* H_dev, float* W_out_dev, uint8_t* mask_dev,
                             void* ws, size_t ws_bytes, pwp_stats* stats_dev, void* stream);

/* One layer end to end from host memory, the transfers overlapping the work.
 *   W_host, X_host  : pinned host copies of W (c x b, wtype) and X ([n, b], xtype).
 *   W_dev, X_dev    : device buffers of the same sizes (overwritten with the copies).
 *   H_dev           : b x b fp32 device scratch (as pwp_prune_layer_x; may be NULL for
 *                     PWP_WANDA and PWP_MAGNITUDE).
 *   W_out_dev, mask_dev : device results, as pwp_prune_layer.
 *   W_out_host, mask_out_host : pinned host buffers (c x b fp32, c x b bytes) receiving
 *                     copies of the results.
 * X goes in in row chunks on a copy stream of the call's own, each chunk folded into H as
 * soon as it lands (the fp32 sum over chunks rounds like any other split of the tokens);
 * W follows while H is factored; with PWP_THANOS and PWP_SPARSEGPT (alpha 0) every column
 * block of W-hat and of the mask goes back as soon as the sweep has finished it (its update
 * and its removals applied), the rest at the end.  The work is enqueued on `stream`, which
 * waits for the last copy: once it is synchronised, the host outputs are complete.  Errors
 * as pwp_prune_layer_x. */
pwp_status pwp_prune_layer_host(const pwp_config* cfg, const void* W_host, int32_t wtype,
                                int32_t c, int32_t b, const void* X_host, int32_t xtype,
                                int64_t n, void* W_dev, void* X_dev, float* H_dev,
                                float* W_out_dev, uint8_t* mask_dev, float* W_out_host,
                                uint8_t* mask_out_host, void* ws, size_t ws_bytes,
                                pwp_stats* stats_dev, void* stream);

/* A sequence of same-shaped layers end to end from host memory (a model pruned layer by
 * layer), each layer's transfers overlapping its neighbours' work: layer i+1's X and W go
 * in on an input copy stream while layer i is pruned, and layer i's results come back on
 * an output copy stream while layer i+1 is.  Per layer the steps and results are those of
 * pwp_prune_layer_host (X in row chunks folded into H as they land, finished column blocks
 * returned during the sweep), each layer against its own H.
 *   nlayers         : number of layers (0: nothing to do).
 *   W_host[i], X_host[i] : pinned host copies of layer i's W (c x b, wtype) and X ([n, b],
 *                     xtype); every layer has the same c, b, n and types.
 *   W_out_host[i], mask_out_host[i] : pinned host buffers (c x b fp32, c x b bytes).
 *   dev, dev_bytes  : device scratch of at least pwp_layers_host_bytes(...) bytes, 256-byte
 *                     aligned (two input and two output buffers, H and the prune workspace).
 *   stats_dev       : nlayers pwp_stats records in device memory, one per layer.
 * The work is enqueued on `stream`, which waits for the last copy: once it is synchronised
 * every host output is complete.  Errors as pwp_prune_layer_x (PWP_EWORKSPACE when dev is
 * missing, misaligned or too small); a layer's own failure is in its stats record. */
size_t pwp_layers_host_bytes(const pwp_config* cfg, int32_t c, int32_t b, int64_t n, int32_t wtype,
                             int32_t xtype);
pwp_status pwp_prune_layers_host(const pwp_config* cfg, int32_t nlayers, const void* const* W_host,
                                 int32_t wtype, int32_t c, int32_t b, const void* const* X_host,
                                 int32_t xtype, int64_t n, float* const* W_out_host,
                                 uint8_t* const* mask_out_host, void* dev, size_t dev_bytes,
                                 pwp_stats* stats_dev, void* stream);

/* Stepwise sweep: one layer's rows sharded over ranks (one process per GPU), pruned with the
 * unstructured budget counted over all ranks' rows ("Pruning LLMs with Thanos", section
 * "Contribution two: keep the budget global and the execution local": the budget couples
 * rows only through each block's threshold; section "The layer-reconstruction lens": the
 * rest of the work is per row).  The caller drives the block loop of pwp_prune_layer and,
 * between the steps, combines three buffers over ranks (pwp_sweep_buffers):
 *   for t = 0 .. nblk-1 (nblk = ceil(b / block)):
 *     SCORE(t)       block t-1's update and block t's scores (level-1 histogram, and the
 *                    level-2 one of the predicted bin); this rank's removal count appended
 *     -> sum `level1` over ranks (uint32, in place)
 *     PICK_BIN(t)    the level-1 bin of the residual budget's last key
 *     REREAD(t)      this rank's level-2 counts when the bin was not predicted
 *     -> sum `level2` over ranks
 *     PICK_KEY(t)    the exact threshold and the number of tied entries taken
 *     COUNT_TIES(t)  this rank's tied entries per block column
 *     -> gather `ties` from every rank into ties_all (world x 128 uint32, rank order)
 *     CUT_TIES(t)    this rank's share of the ties, in (column, row) order with lower ranks'
 *                    rows first
 *     SOLVE(t)       the masks and joint solves of this rank's rows
 *   then FINISH (the last update; stats_dev->pruned = this rank's removals, no budget
 *   check).  SETUP comes first (stats, W-hat, the factor of H, the inverse rows).
 * All ranks must pass the same cfg, b, c_total and H (the layer's whole undamped 2XX^T,
 * destroyed as by pwp_prune_layer).  Thanos and SparseGPT, pattern PWP_UNSTRUCTURED,
 * alpha 0 (other patterns need no exchange: prune row slices with pwp_prune_layer);
 * c_total * b < 2^31.  With world = 1 the steps reproduce pwp_prune_layer exactly.  The
 * workspace is pwp_workspace_bytes(cfg, c, b); the same one for every step of a sweep. */
typedef enum {
    PWP_SWEEP_SETUP = 0, PWP_SWEEP_SCORE = 1, PWP_SWEEP_PICK_BIN = 2, PWP_SWEEP_REREAD = 3,
    PWP_SWEEP_PICK_KEY = 4, PWP_SWEEP_COUNT_TIES = 5, PWP_SWEEP_CUT_TIES = 6, PWP_SWEEP_SOLVE = 7,
    PWP_SWEEP_FINISH = 8
} pwp_sweep_step_kind;
typedef struct {
    const pwp_config* cfg;
    const void* W_dev;          /* this rank's rows: c x b, wtype */
    int32_t wtype;
    int32_t c;                  /* this rank's rows */
    int32_t b;
    int64_t c_total;            /* every rank's rows: the budget counts these */
    float* H_dev;
    float* W_out_dev;           /* c x b fp32 */
    uint8_t* mask_dev;          /* c x b */
    void* ws;
    size_t ws_bytes;
    pwp_stats* stats_dev;
    const uint32_t* ties_all_dev;   /* world x 128, for PWP_SWEEP_CUT_TIES */
    int32_t world;
    int32_t rank;
    void* stream;
} pwp_sweep;
pwp_status pwp_sweep_step(const pwp_sweep* sweep, int32_t step, int32_t t);
/* Device addresses (inside ws) and lengths (uint32 words) of the buffers exchanged between
 * steps: level1 (summed), level2 (summed), ties (this rank's, to gather). */
pwp_status pwp_sweep_buffers(const pwp_sweep* sweep, uint32_t** level1, int64_t* n_level1, uint32_t** level2,
                             int64_t* n_level2, uint32_t** ties, int64_t* n_ties);

/* Compressed 2:4 storage of a pruned layer ("Weight Pruning in Large Language Models
 * ...", llms.blog, section "N:M Semi-Structured Sparsity (2:4 Pattern)": only the two
 * kept values of every aligned group of four, at 16-bit precision, and 2-bit index
 * metadata are stored).  The pages do not give the metadata layout sparse tensor cores
 * read; this one is plain and row-major:
 *   W_hat_dev : c x b fp32 (e.g. pwp_prune_layer's W_out), 16-byte aligned;
 *   mask_dev  : c x b bytes, 1 = removed, 4-byte aligned; every aligned group of four
 *               must keep exactly two entries (mask 0);
 *   values_dev: c x b/2 uint16, the kept values as bfloat16 bit patterns (round to
 *               nearest even), in column order within each group;
 *   meta_dev  : c x ceil(b/32) uint32; group g of a row is the 4-bit field
 *               idx0 | idx1 << 2 (positions 0..3 of its kept entries, idx0 < idx1) at
 *               bits 4(g%8).. of word g/8 of the row;
 *   1 <= c, 4 <= b <= 16384, b % 4 == 0, c*b < 2^31.
 * stats_dev is cleared first; a group that does not keep exactly two entries sets status
 * PWP_EINVAL (its field then reads positions 0 and 1). */
pwp_status pwp_pack_24(const float* W_hat_dev, const uint8_t* mask_dev, int32_t c, int32_t b,
                       uint16_t* values_dev, uint32_t* meta_dev, pwp_stats* stats_dev, void* stream);

/* Prune without a caller-provided workspace (the pages have no counterpart: this is a
 * convenience of this library).  For callers that cannot allocate device memory when
 * they call -- an operator in a runtime that hands it only its input and output
 * buffers, or a process whose device memory belongs to a framework allocator -- the
 * scratch comes from one static device array of PWP_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads the library keeps until the process exits.
 *   Arguments, results and H's destruction are exactly those of pwp_prune_layer.
 *   Returns PWP_EWORKSPACE, without enqueuing anything, when the configuration needs
 *   more scratch than PWP_NOALLOC_SCRATCH_BYTES (pwp_workspace_bytes tells how much).
 *   The first call on each device looks up the array's device address (with that
 *   device current); make that first call before capturing any stream into a graph.
 *   After cudaDeviceReset the next call looks the address up again (the lookup is
 *   keyed by the context), so it must again come before any capture.
 *   Nothing is allocated or freed.  All calls share the one array: calls whose work
 *   overlaps on the GPU (different streams, or threads without ordering) race and give
 *   wrong results; order them. */
#define PWP_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
pwp_status pwp_prune_layer_noalloc(const pwp_config* cfg, const void* W_dev, int32_t wtype,
                                   int32_t c, int32_t b, float* H_dev, float* W_out_dev,
                                   uint8_t* mask_dev, pwp_stats* stats_dev, void* stream);

/* Instrumentation (no counterpart on the pages).
 * pwp_kernel_launches: number of kernels this process has enqueued through the library.
 * pwp_profile_enable(which, capacity): record a pair of CUDA events on the call's stream
 *   around each launch of kernel class `which` (pwp_kernel_class), for up to `capacity`
 *   launches; which < 0 switches recording off and frees the events.
 * pwp_profile_read(ms, cap): waits for the recorded events, writes up to `cap` elapsed
 *   times (milliseconds, one per launch, in launch order) and returns how many; the
 *   record is then cleared. */
typedef enum {
    PWP_K_HESSIAN = 0,   /* the X X^T accumulation kernel */
    PWP_K_FACTOR = 1,    /* the whole damping + factorisation phase */
    PWP_K_STREAM = 2,    /* per block: trailing update + rescoring + histogram */
    PWP_K_SELECT = 3,    /* per block: exact threshold selection */
    PWP_K_SOLVE = 4,     /* per block: per-row solves and in-block update */
    PWP_K_ROWPRUNE = 5,  /* Wanda / magnitude: the per-row (or per-group) selection */
    PWP_K_COLNORM = 6    /* Wanda from X: the column norms of X */
} pwp_kernel_class;
int64_t pwp_kernel_launches(void);
/* pwp_set_wait_limit(polls): every bounded device-side wait of the tensor-core kernels
 *   (an mbarrier wait between the copy, MMA and epilogue roles of one CTA) gives up after
 *   this many polls and the call reports PWP_ETIMEOUT in stats (status_site names the
 *   kernel).  Applies to kernels enqueued after the call; polls < 0 restores the default
 *   (2^26); 0 makes every such wait give up at once, which lets a test drive the timeout
 *   paths without any fault.  Copies and MMAs already in flight are always waited for
 *   with the default limit before a CTA leaves.  Returns the previous limit.  Process-wide,
 *   not tied to a stream: set it only while no other thread enqueues library work. */
int64_t pwp_set_wait_limit(int64_t polls);
int32_t pwp_profile_enable(int32_t which, int32_t capacity);
int32_t pwp_profile_read(float* ms_out, int32_t cap);

/* Static, NUL-terminated description of a status code. */
const char* pwp_status_string(int32_t status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t pwp_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PWP_H */
