/*
 * wildcat.h -- C ABI of the B200 (sm_100a) WildCat hot path.
 *
 * WildCat approximates softmax attention O = D^-1 A V, A = exp(beta Q K^T),
 * by attending over a weighted coreset of the keys ("WildCat: Near-Linear
 * Attention in Theory and Practice", Schroeder & Mackey, Sec. 2):
 *
 *   select   randomly pivoted Cholesky (RPCholesky) on the key kernel
 *            h(K,K) = exp(beta K K^T) picks r pivot keys S and builds the
 *            partial Cholesky factor F (Sec. 2, "randomly pivoted Cholesky";
 *            Alg. 1 RPNys)
 *   weights  Nystrom weights W = h(K_S,K_S)^+ h(K_S,K) applied to (V, 1_n):
 *            V_S = W V and w = W 1_n, formed as F_S^-T (F^T (V, 1_n))
 *            (Sec. 2 plug-in estimator; Alg. 2 CompressKV)
 *   attend   O_hat = diag(U w)^-1 U V_S, U = exp(beta Q K_S^T), each entry
 *            clipped to the value range [v_min j, v_max j] of V
 *            (Sec. 2, value-range clip; Alg. 3 WtdAttn); bf16 inputs with
 *            d in {64, 128} run on the tensor cores (tcgen05, fp32
 *            accumulation in tensor memory; P and V_S rounded to bf16 for
 *            the numerator's products, the denominator sum_l P_l w_l in fp32
 *            from the unrounded P); other inputs on CUDA cores in fp32
 *   forward  the three stages back to back (Alg. 4, the WildCat module)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - An "instance" is one (batch, head) pair; BH instances are independent
 *    and are stored one after another (instance b = batch * H + head).
 *  - All tensors are dense, row-major and contiguous.  Q is [BH, m, d];
 *    K and V are [BH, n, d]; their dtype is WILDCAT_F32 or WILDCAT_BF16.
 *    Every other tensor has a fixed type given below.
 *  - The factor F is float32 [BH, r, n]: F[b, i, l] is entry l of factor
 *    column i, so each column is contiguous over the n keys.
 *  - Unless a name ends in _host, every pointer is a DEVICE pointer owned by
 *    the caller.  The library keeps no pointer after a call returns, and no
 *    call allocates device memory: scratch space is the caller's
 *    `workspace` (size from the matching *_workspace_size query, 256-byte
 *    aligned).  (The forwards create, on first use per device, one library
 *    stream and a few events; wildcat_attend_noalloc uses a static array.)
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; a call returns once its kernels are launched.
 *  - Argument checks happen on the host before anything is launched and
 *    return WILDCAT_ERR_INVALID_ARG / WILDCAT_ERR_UNSUPPORTED with no work
 *    enqueued.  A failed launch returns WILDCAT_ERR_CUDA.  In every error
 *    case wildcat_last_error() (per thread) describes the failure.
 *  - Supported head dims: d in {32, 64, 128}.  Device pointers to Q, K, V,
 *    K_S must be 16-byte aligned.
 *  - An instance whose pivots run out before r (total residual mass zero,
 *    or a pivot residual g_s <= eps, the truncation that stands in for the
 *    pseudo-inverse) has effective rank r' < r.  That is not an error: the
 *    rank is reported, S holds -1 past r', and F, K_S, V_S and w hold zeros
 *    there.
 *  - Pivot draws: uniform u_i of step i for instance b is Philox4x32-10
 *    (Salmon et al., SC'11) with key (seed_lo, seed_hi) and counter
 *    (i, inst0 + b, 0, 0); u = (x + 1) * 2^-53 where x is the top 53 bits of
 *    the 64-bit word (x1:x0).  The pivot is the first key whose cumulative
 *    residual diagonal reaches u * T, T the total residual mass.  inst0 is
 *    the global index of the call's first instance: a batch split into
 *    shards (e.g. one per GPU) draws exactly the pivots of the whole batch
 *    when each shard passes its offset.
 */
#ifndef WILDCAT_H_
#define WILDCAT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WILDCAT_OK = 0,
    WILDCAT_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment */
    WILDCAT_ERR_UNSUPPORTED = 2, /* valid but not implemented (head dim, size limit) */
    WILDCAT_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    WILDCAT_ERR_WORKSPACE = 4,   /* workspace too small or misaligned */
    WILDCAT_ERR_TIMEOUT = 5      /* a kernel's bounded wait expired (see wildcat_get_device_status) */
} wildcat_status;

typedef enum { WILDCAT_F32 = 0, WILDCAT_BF16 = 1 } wildcat_dtype;

/* Library version (major * 10000 + minor * 100 + patch). */
int wildcat_version(void);

/* Message for the last failed call on this thread ("" if none). */
const char* wildcat_last_error(void);

/* Static name of a status code. */
const char* wildcat_status_string(int status);

/*
 * wildcat_select -- RPCholesky coreset selection (Sec. 2, randomly pivoted
 * Cholesky; Alg. 1 RPNys).  For every instance, r sequential steps: draw the
 * pivot s from the residual diagonal, form the factor column
 * F[:, i] = g / sqrt(g_s), g = h(K, k_s) - F[:, :i] F[s, :i]^T, and update the
 * residual diagonal d <- max(d - F[:, i]^2, 0), d_s = 0.  The kernel is
 * evaluated as exp(beta (<x, y> - M_K)), M_K = max_l |k_l|^2, a constant
 * factor that leaves pivots and weights unchanged.
 *
 *   K      [BH, n, d] keys, dtype `dtype`
 *   beta   kernel inverse temperature (> 0, finite)
 *   r      coreset size, 1 <= r <= n
 *   seed   64-bit Philox key of the pivot draws
 *   inst0  global index of instance 0 of this call (0 unless sharded), >= 0
 *   eps    truncation threshold (relative to max_l h(k_l, k_l)), >= 0
 *   S      out [BH, r] int32 pivot indices in draw order, -1 past the rank
 *   F      out [BH, r, n] float32 factor
 *   rank   out [BH] int32 effective rank r'
 *   K_S    out [BH, r, d] gathered pivot keys (dtype `dtype`), or NULL
 */
wildcat_status wildcat_select(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta,
                              int r, uint64_t seed, int64_t inst0, float eps, int32_t* S, float* F,
                              int32_t* rank, void* K_S, void* stream);

/*
 * wildcat_select_ws -- wildcat_select with a workspace (>= wildcat_select_
 * workspace_size(BH, n) bytes, 256-byte aligned, owned by the caller).  With
 * it the library may run the global-sync form of the select kernel: when
 * there are few instances (BH well below the SM count) each instance gets
 * up to 32 CTAs that meet at a counter barrier in the workspace instead of
 * a thread-block cluster (clusters of 16 CTAs must share one GPC, so few fit
 * at once).  The grid is launched cooperatively (all CTAs co-resident); every
 * barrier wait is bounded (2 s, WILDCAT_ERR_TIMEOUT in the device status
 * word on expiry).  Results equal wildcat_select's to float32 rounding.
 * The workspace also enables phases for long coresets (r >= 512, BH at most
 * the SM count): the steps run as launches of 64 steps; between
 * them each instance still going keeps its residual diagonal in the
 * workspace, and the next launch (global sync over the whole GPU) gives each
 * such instance about SMs / (instances still going) CTAs (at least 256 key
 * rows each, up to 160 CTAs).  The
 * instances whose factor truncated early no longer leave the longest ones on
 * the few CTAs of the first launch.  workspace may be NULL (then exactly
 * wildcat_select).  wildcat_forward* carve this workspace from theirs.
 */
size_t wildcat_select_workspace_size(int64_t BH, int64_t n);
wildcat_status wildcat_select_ws(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta,
                                 int r, uint64_t seed, int64_t inst0, float eps, int32_t* S,
                                 float* F, int32_t* rank, void* K_S, void* workspace,
                                 size_t ws_bytes, void* stream);

/*
 * wildcat_select_fixed -- the same factorisation with the pivots given
 * (test entry point: lets the device path run on the oracle's pivots).
 * S_fixed [BH, r] int32; a negative or out-of-range entry ends that
 * instance's factorisation (rank = its position).  S (out, may be NULL)
 * receives the pivots actually used.  Other arguments as wildcat_select.
 */
wildcat_status wildcat_select_fixed(const void* K, int dtype, int64_t BH, int64_t n, int d,
                                    float beta, int r, float eps, const int32_t* S_fixed,
                                    int32_t* S, float* F, int32_t* rank, void* K_S, void* stream);

/*
 * wildcat_weights -- Nystrom weights applied to (V, 1_n) (Sec. 2 plug-in
 * estimator: W multiplies (V, 1_n) before the queries; Alg. 2 CompressKV).
 * Y = F^T (V, 1_n) is reduced over the n keys, then F_S^T X = Y is solved by
 * back substitution with F_S[a, j] = F[b, j, S[a]] (lower triangular in
 * pivot order; entries above the diagonal are ignored).
 *
 *   F, S, rank   from wildcat_select
 *   V            [BH, n, d] values, dtype `dtype`
 *   V_S          out [BH, r, d] float32, rows of W V (zero past the rank)
 *   w            out [BH, r] float32, W 1_n (zero past the rank)
 *   vmin, vmax   out [BH, d] float32 column-wise range of V
 *   workspace    >= wildcat_weights_workspace_size(BH, n, d, r) bytes
 */
size_t wildcat_weights_workspace_size(int64_t BH, int64_t n, int d, int r);
wildcat_status wildcat_weights(const float* F, const int32_t* S, const int32_t* rank,
                               const void* V, int dtype, int64_t BH, int64_t n, int d, int r,
                               float* V_S, float* w, float* vmin, float* vmax, void* workspace,
                               size_t ws_bytes, void* stream);

/*
 * wildcat_weights_inverse -- the same outputs as wildcat_weights, through the
 * inverse that RPNys maintains (Sec. 2): h(K_S, K_S)^-1 is grown pivot by
 * pivot with the rank-one update (y = H_S^-1 b, sc = h(k_s, k_s) - b.y,
 * H_S'^-1 = [[H_S^-1, 0], [0, 0]] + g g^T, g = (y, -1) / sqrt(sc)), then
 * W (V, 1_n) = H_S^-1 h(K_S, K) (V, 1_n).  Equal to the factor route in exact
 * arithmetic; provided to compare the two numerically.  fp64 arithmetic
 * throughout from the inputs widened exactly; V_S and w are rounded to
 * float32 at the end.  h carries the shift M = max_l |k_l|^2, which cancels.
 *
 *   K, V   [BH, n, d] keys and values, dtype `dtype`
 *   S      [BH, r] int32 pivots in selection order; S[b, a] in [0, n) for
 *          a < rank[b] (as written by wildcat_select; not checked on the device)
 *   rank   [BH] int32 effective ranks, 0 <= rank[b] <= r
 *   beta   the kernel's beta (> 0)
 *   V_S, w, vmin, vmax   outputs as wildcat_weights (rows >= rank[b] zero)
 *   workspace >= wildcat_weights_inverse_workspace_size(BH, n, d, r) bytes,
 *          256-byte aligned; about 16 BH r^2 bytes (two r x r fp64 arrays)
 * Returns WILDCAT_ERR_UNSUPPORTED for r > 2048 (the size query returns 0).
 */
size_t wildcat_weights_inverse_workspace_size(int64_t BH, int64_t n, int d, int r);
wildcat_status wildcat_weights_inverse(const void* K, const void* V, int dtype, const int32_t* S,
                                       const int32_t* rank, int64_t BH, int64_t n, int d, int r,
                                       float beta, float* V_S, float* w, float* vmin, float* vmax,
                                       void* workspace, size_t ws_bytes, void* stream);

/*
 * wildcat_attend -- weighted-coreset attention (Alg. 3 WtdAttn):
 *   u_il = exp(beta <q_i, k_S_l> - beta M_Q),  M_Q = max_i |q_i| * max_l |k_S_l|
 *   O_hat_ij = fminf(fmaxf(sum_l u_il V_S[l, j] / sum_l u_il w_l, vmin_j), vmax_j)
 * The shift M_Q (one per instance) keeps every u_il <= 1 and cancels in the
 * ratio; the tensor-core path (bf16, d in {64, 128}) shifts each query row by
 * beta |q_i| max_l |k_S_l| instead, which cancels in the same way.  A normaliser that is zero or negative (Nystrom weights have mixed
 * signs) is not special-cased: the ratio is clipped as is, and a NaN ratio
 * (0/0) becomes vmin_j.
 *
 *   Q      [BH, m, d] queries, dtype `dtype`
 *   K_S    [BH, r, d] pivot keys, dtype `dtype`
 *   rank   [BH] int32 effective ranks (only the first rank[b] rows are used)
 *   V_S, w, vmin, vmax   from wildcat_weights
 *   O      out [BH, m, d] float32
 *   workspace >= wildcat_attend_workspace_size(BH, m, d, r) bytes
 */
size_t wildcat_attend_workspace_size(int64_t BH, int64_t m, int d, int r);
wildcat_status wildcat_attend(const void* Q, const void* K_S, int dtype, int64_t BH, int64_t m,
                              int d, int r, const int32_t* rank, float beta, const float* V_S,
                              const float* w, const float* vmin, const float* vmax, float* O,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * wildcat_decode_attend -- KV-cache decode with new tokens (Sec. 2: after
 * CompressKV, m new tokens cost O(rmd + m^2 d)).  New query i attends over
 * the compressed cache (K_S, V_S, w from select/weights) and, exactly, over
 * the new tokens j <= i (causal):
 *   N_i = sum_l u_il V_S[l] + sum_{j<=i} e_ij V_new[j],  D_i = sum_l u_il w_l + sum_{j<=i} e_ij,
 *   u_il = exp(beta <q_i, k_S_l> - beta M), e_ij = exp(beta <q_i, k_new_j> - beta M),
 *   M = max_i |q_i| * max(max_l |k_S_l|, max_j |k_new_j|) per instance,
 *   O_i = clip(N_i / D_i) to the range of the cache (vmin, vmax) and V_new.
 *
 *   Q_new, K_new, V_new  [BH, m, d] new tokens, dtype `dtype`
 *   K_S, rank, V_S, w, vmin, vmax   the compressed cache
 *   O      out [BH, m, d] float32
 *   workspace >= wildcat_decode_attend_workspace_size(BH, d) bytes
 */
size_t wildcat_decode_attend_workspace_size(int64_t BH, int d);
wildcat_status wildcat_decode_attend(const void* Q_new, const void* K_new, const void* V_new,
                                     const void* K_S, int dtype, int64_t BH, int64_t m, int d, int r,
                                     const int32_t* rank, float beta, const float* V_S,
                                     const float* w, const float* vmin, const float* vmax,
                                     float* O, void* workspace, size_t ws_bytes, void* stream);

/*
 * wildcat_attend_noalloc -- wildcat_attend for callers that cannot allocate
 * device memory.  The paper has no counterpart; this is a deployment
 * convenience.  Such callers only hold pointers handed to them by another
 * component that owns the GPU's memory (for example a serving engine that
 * reserves nearly all of it for its KV cache), or run in a loop where a
 * cudaMalloc, which can synchronise the device, is not acceptable, so they
 * cannot supply the `workspace` that wildcat_attend needs.
 *
 * Same arguments and result as wildcat_attend, without workspace.  The
 * caller still provides every input and the output O.  The call allocates
 * nothing: its scratch is a static device array of
 * WILDCAT_NOALLOC_SCRATCH_BYTES (1 MiB) that every GPU loading this library
 * holds until the process exits.  Sizes needing more than that, about
 * 4 * BH * (min(64, ceil(m / 1024)) + 1) bytes, return
 * WILDCAT_ERR_UNSUPPORTED before anything is launched.
 *
 * The first call on each device looks up the array's device address (a
 * host-side runtime query, no allocation); make that first call before any
 * stream capture.  The address is remembered per device ordinal for the
 * life of the process: it assumes the device's primary context is the one
 * in use throughout, so after cudaDeviceReset (or with another context made
 * current on that ordinal) the remembered address is stale and this entry
 * point must not be called again in that process.  The call launches on the
 * current device; every pointer must belong to it.  All calls share the one array, so calls whose work
 * overlaps on the GPU (e.g. on two streams) race and must be serialised by
 * the caller.  Each call writes every scratch word before reading it, so
 * the contents left by an earlier call do not matter.
 */
#define WILDCAT_NOALLOC_SCRATCH_BYTES (1u << 20)
wildcat_status wildcat_attend_noalloc(const void* Q, const void* K_S, int dtype, int64_t BH,
                                      int64_t m, int d, int r, const int32_t* rank, float beta,
                                      const float* V_S, const float* w, const float* vmin,
                                      const float* vmax, float* O, void* stream);

/*
 * wildcat_forward -- the whole module (Alg. 4): select -> weights -> attend,
 * on `stream`, with every intermediate in `workspace`.  seed, inst0 and eps
 * as in wildcat_select.  The value range of V (needed only by the attend)
 * runs on a library-owned stream of the current device, forked from `stream`
 * before the select and joined back before the attend, so it overlaps the
 * select; the same holds for wildcat_forward_ex / _binned / _host /
 * _ex_host.  A per-device lock covers each call's fork-to-join section, so
 * calls from several threads are correct (their value ranges serialize).
 *
 *   Q [BH, m, d], K and V [BH, n, d] (dtype `dtype`); O out [BH, m, d] float32
 *   S_out [BH, r] int32 and rank_out [BH] int32: optional outputs (or NULL);
 *     when given, the select writes them in place and the weights and attend
 *     stages read them from there, so they must not overlap any other argument
 *   workspace >= wildcat_forward_workspace_size(BH, m, n, d, r, dtype) bytes
 */
size_t wildcat_forward_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype);
wildcat_status wildcat_forward(const void* Q, const void* K, const void* V, int dtype, int64_t BH,
                               int64_t m, int64_t n, int d, float beta, int r, uint64_t seed,
                               int64_t inst0, float eps, float* O, int32_t* S_out,
                               int32_t* rank_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Options of wildcat_forward_ex (Sec. 2: divide-and-conquer bins, recentring
 * of the keys and temperature rescaling).
 *   nbins     >= 1: keys cut into nbins contiguous bins (see
 *             wildcat_forward_binned); 1 = no binning
 *   recenter  0 or 1: select and weight the coreset on the recentred keys
 *             k_l - kbar, kbar the instance's mean key (softmax attention is
 *             unchanged by the shift)
 *   tau       > 0: temperature; the coreset is selected and weighted with
 *             the key kernel exp(beta <x, y> / tau^2), i.e. on keys K / tau,
 *             while queries become tau Q, leaving attention unchanged.  The
 *             pages' closed form for tau (their eq. 12) did not survive, so
 *             tau is the caller's; 1 = no rescaling.
 * The attend step needs neither: with the original pivot keys and beta, the
 * recentring shift and 1 / tau cancel in N / D.
 */
typedef struct {
    int nbins;
    int recenter;
    float tau;
} wildcat_options;

/*
 * wildcat_forward_ex -- wildcat_forward with wildcat_options (NULL: the
 * defaults {1, 0, 1}, identical to wildcat_forward).  S_out [BH, r] global
 * key indices and rank_out [BH, nbins] as in wildcat_forward_binned.
 *   workspace >= wildcat_forward_ex_workspace_size(...) bytes
 */
size_t wildcat_forward_ex_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype,
                                         const wildcat_options* opts);
wildcat_status wildcat_forward_ex(const void* Q, const void* K, const void* V, int dtype, int64_t BH,
                                  int64_t m, int64_t n, int d, float beta, int r, uint64_t seed,
                                  int64_t inst0, float eps, const wildcat_options* opts, float* O,
                                  int32_t* S_out, int32_t* rank_out, void* workspace,
                                  size_t ws_bytes, void* stream);

/*
 * wildcat_forward_binned -- the module with divide-and-conquer binning
 * (Sec. 2: B bins, r / B pivots each, selected in parallel).  The n keys of
 * every instance are cut into nbins contiguous bins of n / nbins keys; bin q
 * gets its own RPCholesky coreset of r / nbins pivots (pivot draws use the
 * instance index (inst0 + b) * nbins + q) and its own Nystrom weights over
 * its own keys (block-diagonal W).  The output attends over the union of the
 * bins' coresets; the value range is over all n keys.  n and r must be
 * multiples of nbins; nbins = 1 is wildcat_forward.  Same as
 * wildcat_forward_ex with options {nbins, 0, 1}.
 *
 *   S_out    [BH, r] int32 global key index of every union row, -1 past a
 *            bin's rank (or NULL); row q * (r / nbins) + a is bin q's a-th pivot
 *   rank_out [BH, nbins] int32 effective rank of every bin (or NULL)
 *   workspace >= wildcat_forward_binned_workspace_size(...) bytes
 */
size_t wildcat_forward_binned_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r,
                                             int nbins, int dtype);
wildcat_status wildcat_forward_binned(const void* Q, const void* K, const void* V, int dtype,
                                      int64_t BH, int64_t m, int64_t n, int d, float beta, int r,
                                      int nbins, uint64_t seed, int64_t inst0, float eps, float* O,
                                      int32_t* S_out, int32_t* rank_out, void* workspace,
                                      size_t ws_bytes, void* stream);

/*
 * wildcat_forward_host -- wildcat_forward on HOST buffers: copies Q, K, V
 * from host memory into the device workspace, runs the forward, copies O
 * (and optionally S, rank) back, and waits for the stream.  K is copied
 * first on a library-owned copy stream; V and Q follow while the select
 * runs on `stream`, and the weights and attend stages wait for them.  Calls
 * on one device are serialized (a per-device lock guards the copy stream).
 * Host buffers should be page-locked for full copy bandwidth.
 *
 *   Q_host, K_host, V_host   host input arrays (layouts as wildcat_forward)
 *   O_host                   host output [BH, m, d] float32
 *   S_host, rank_host        optional host outputs (or NULL)
 *   workspace >= wildcat_forward_host_workspace_size(...) bytes (device)
 */
size_t wildcat_forward_host_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r,
                                           int dtype);
wildcat_status wildcat_forward_host(const void* Q_host, const void* K_host, const void* V_host,
                                    int dtype, int64_t BH, int64_t m, int64_t n, int d,
                                    float beta, int r, uint64_t seed, int64_t inst0, float eps,
                                    float* O_host, int32_t* S_host, int32_t* rank_host,
                                    void* workspace, size_t ws_bytes, void* stream);

/*
 * wildcat_forward_ex_host -- wildcat_forward_ex on HOST buffers, pipelined
 * like wildcat_forward_host: K is copied first on the library's copy stream
 * (the recentring mean and the select need only K), V and Q follow while the
 * select runs, the weights stage waits for V and the attend for Q; then O
 * (and optionally S, rank) are copied back and the stream is waited for.
 * Options as in wildcat_forward_ex (NULL: the plain forward).
 *
 *   Q_host, K_host, V_host   host input arrays (layouts as wildcat_forward)
 *   O_host                   host output [BH, m, d] float32
 *   S_host [BH, r] int32, rank_host [BH, nbins] int32: optional host outputs
 *                            as in wildcat_forward_ex (or NULL)
 *   workspace >= wildcat_forward_ex_host_workspace_size(...) bytes (device)
 */
size_t wildcat_forward_ex_host_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r,
                                              int dtype, const wildcat_options* opts);
wildcat_status wildcat_forward_ex_host(const void* Q_host, const void* K_host,
                                       const void* V_host, int dtype, int64_t BH, int64_t m,
                                       int64_t n, int d, float beta, int r, uint64_t seed,
                                       int64_t inst0, float eps, const wildcat_options* opts,
                                       float* O_host, int32_t* S_host, int32_t* rank_host,
                                       void* workspace, size_t ws_bytes, void* stream);

/*
 * wildcat_pivot_uniforms -- the pivot uniforms the select kernels draw
 * (test entry point): u[b, i] for b < BH, i < steps (instance offset 0), as
 * float64, written to the device array u [BH, steps].
 */
wildcat_status wildcat_pivot_uniforms(uint64_t seed, int64_t BH, int steps, double* u,
                                      void* stream);

/*
 * wildcat_get_device_status -- waits for `stream`, then reports and clears
 * the device status words of the current device.  Kernels that wait on
 * mbarriers (the tensor-core weights and attend) or on counters (the select's
 * global-sync form) bound
 * every wait by a time limit; when one expires the kernel records
 * WILDCAT_ERR_TIMEOUT there, stops issuing work, waits (bounded) for its
 * copies in flight, releases its tensor memory and returns, leaving its
 * output incomplete (the select stops every CTA of the instance at the same
 * step and reports the steps taken as the rank).
 * Returns WILDCAT_OK, WILDCAT_ERR_TIMEOUT, or WILDCAT_ERR_CUDA if the stream
 * or the status word could not be read.
 */
wildcat_status wildcat_get_device_status(void* stream);

/*
 * wildcat_test_force_wait_timeout -- test hook for the bounded waits.  With
 * nanoseconds > 0 every later tensor-core attend launch first waits that long
 * on a barrier phase that nothing completes, records WILDCAT_ERR_TIMEOUT in
 * the device status word, releases its tensor memory and returns without
 * writing O.  0 turns the hook off.  Process-wide; for tests only.
 * Returns WILDCAT_ERR_INVALID_ARG outside [0, 1e9].
 */
wildcat_status wildcat_test_force_wait_timeout(int64_t nanoseconds);

/*
 * wildcat_test_force_select_timeout -- test hook for the bounded waits of
 * the select's global-sync form.  With nanoseconds > 0, CTA 0 of every
 * instance never arrives at the third counter barrier and every wait there
 * ends after `nanoseconds` (every instance stops after one step).  The
 * expiry is handled like any other: WILDCAT_ERR_TIMEOUT in the device status
 * word.  0 turns the hook off.  Process-wide; for tests only.  Returns
 * WILDCAT_ERR_INVALID_ARG outside [0, 1e9].
 */
wildcat_status wildcat_test_force_select_timeout(int64_t nanoseconds);

/*
 * wildcat_set_select_kernel -- which form of the select kernel
 * wildcat_select* launch: 0 (default) the global-sync form when a workspace
 * is given and that form has less work per CTA, else clusters; 1 clusters
 * only; 3 the global-sync form wherever a workspace is given and all CTAs
 * fit at once.  Both forms compute the same factorisation (results agree to
 * float32 rounding).  Process-wide; not thread-safe against concurrent
 * select calls.  Returns WILDCAT_ERR_INVALID_ARG for other values.
 */
wildcat_status wildcat_set_select_kernel(int kernel);

/* The form of the select kernel the last select launch on this thread used:
 * 1 clusters, 3 global sync, 0 if none. */
int wildcat_last_select_kernel(void);

/* Threads per CTA of the last select launch on this thread: 512, or 256 when
 * the automatic choice put two CTAs on each SM (twice the cluster size, half
 * the rows per CTA; resident keys only).  0 if none. */
int wildcat_last_select_threads(void);

/*
 * wildcat_set_select_phase_steps -- steps per launch of a select call that
 * has a workspace (wildcat_select_ws and the forward calls): 0 (default)
 * automatic, 64 when r >= 512 and a single launch otherwise; > 0
 * that many steps per launch for any r (the phases apply where the
 * workspace, BH <= SM count and n % 4 == 0 allow them); < 0 always one
 * launch.  Results do not depend on it beyond float32 rounding of the
 * search sums.  Process-wide; not thread-safe against concurrent select
 * calls.  Always returns WILDCAT_OK.
 */
wildcat_status wildcat_set_select_phase_steps(int steps);

/* Launches of the last select call on this thread (1 = no phases), 0 if none. */
int wildcat_last_select_phases(void);

/*
 * wildcat_set_stage_events -- optional stage markers for timing the stages of
 * a forward: every later wildcat_forward, wildcat_forward_ex,
 * wildcat_forward_binned or wildcat_forward_host call on this thread records
 * `after_select` on its stream right after the select's launches and
 * `after_weights` right after the weights' launches, so that the caller can
 * split one timed call into select, weights and attend with
 * cudaEventElapsedTime.  Both are cudaEvent_t handles passed as void*,
 * created and owned by the caller, and must stay valid while calls record
 * them; NULL turns a marker off (the default).  Thread-local.  A failed
 * record is reported as WILDCAT_ERR_CUDA by the forward call.  Always
 * returns WILDCAT_OK.
 */
wildcat_status wildcat_set_stage_events(void* after_select, void* after_weights);

/*
 * wildcat_set_select_cluster -- tuning knob for wildcat_select*: number of
 * CTAs (a thread-block cluster, 1..16, power of two) that share one
 * instance.  0 restores the automatic choice: the G with the least
 * ceil(BH / clusters that fit at once) * ceil(n / G), from the occupancy
 * API (a 16-CTA cluster needs 16 SMs of one GPC, so few of them fit).  Process-wide; not thread-safe
 * against concurrent select calls.  Returns WILDCAT_ERR_INVALID_ARG for
 * other values.
 */
wildcat_status wildcat_set_select_cluster(int ctas_per_instance);

/* The cluster size the last select launch on this thread used (0 if none). */
int wildcat_last_select_cluster(void);

#ifdef __cplusplus
}
#endif

#endif /* WILDCAT_H_ */
