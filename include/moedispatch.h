/*
 * moedispatch.h -- C ABI of libmoedispatch, the B200 (sm_100a) MoE token
 * dispatch / combine path for expert parallelism.
 *
 * The problem follows the pages' statement of one expert-parallel dispatch
 * ("AllToAllDispatchScenario", mlsysim API page: total_tokens of hidden_dim
 * values over n_devices holding n_experts):
 *   T tokens (total_tokens), H hidden values each (hidden_dim, bf16),
 *   E experts (n_experts) placed on R ranks (n_devices) by expert_to_rank,
 *   each token routed to its top-k experts.
 * The R ranks are virtual: they are partitions of one GPU's memory, so every
 * "send" is a row copy inside HBM and there are no collectives.  Source rank
 * of token t is src(t) = t / (T / R): each rank routes a contiguous block of
 * T/R tokens ("DODOCO: MoE AlltoAll Traffic Matrices on Real Text", Setup).
 *
 * Conventions for every entry point below:
 *   - Pointers are DEVICE pointers unless marked host; the caller allocates
 *     and owns all memory.  The library never allocates or frees.
 *   - Arrays are dense, row-major, without padding.  bf16 is the IEEE
 *     bfloat16 bit pattern (__nv_bfloat16).  x, y, out, z must be 16-byte
 *     aligned and H must be a multiple of 8 (16-byte rows).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Each call
 *     only enqueues work on it and returns; results are ready when the
 *     stream reaches that point.  As for any CUDA runtime launch, the device
 *     that holds the pointers and the stream must be the calling thread's
 *     current device.
 *   - The return value reports what can be checked on the host: MD_ERR_ARG
 *     for bad sizes or pointers, MD_ERR_WORKSPACE for a short workspace,
 *     MD_ERR_CUDA when a launch fails.  Nothing is enqueued on an error.
 *   - `dev_status` (device int32, may be NULL) receives what only the data
 *     can show: an expert index outside [0, E), an expert twice in one
 *     token's list, a placement that does not give every rank E/R experts,
 *     a row index outside its buffer (MD_ERR_DATA), or a bounded wait that
 *     ran out (MD_ERR_TIMEOUT).  Each call that takes it sets it to MD_OK
 *     first; read it after synchronising.  Offending entries are skipped,
 *     never written out of bounds; the other outputs are then unspecified.
 *   - Calls that share a workspace, or write the same outputs, must not run
 *     concurrently.
 */
#ifndef MOEDISPATCH_H
#define MOEDISPATCH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum md_status {
    MD_OK = 0,
    MD_ERR_ARG = 1,
    MD_ERR_UNSUPPORTED = 2,
    MD_ERR_CUDA = 3,
    MD_ERR_WORKSPACE = 4,
    MD_ERR_DATA = 5,
    MD_ERR_TIMEOUT = 6
} md_status;

#define MD_CONV 0              /* one row per (token, expert) assignment   */
#define MD_DEDUP 1             /* one row per distinct (token, rank) pair  */
#define MD_GATE_TOPK_SOFTMAX 0 /* softmax over the k selected logits       */
#define MD_GATE_FULL_SOFTMAX 1 /* softmax over all E logits, then gathered */
#define MD_COMBINE_FUSED 0     /* one weighted sum per token               */
#define MD_COMBINE_WIRE 1      /* per-rank partial sums (bf16), then sum   */
#define MD_SEED_CONTIGUOUS 0   /* placement search starts contiguous       */
#define MD_SEED_GREEDY_PAIRS 1 /* placement search starts from greedy pairs*/
#define MD_MAX_PAIR_EXPERTS 256 /* pair counts are E^3 entries               */
#define MD_REFINE_NONE 0       /* placement: seed only                      */
#define MD_REFINE_SWAPS 1      /* best positive single swaps                */
#define MD_REFINE_KL 2         /* Kernighan-Lin passes                      */

#define MD_MAX_TOPK 32
#define MD_MAX_EXPERTS 1024
#define MD_MAX_RANKS 64

/* Name of a status code; never NULL. */
const char *md_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int md_version(void);

/* Number of kernels this library has launched in this process so far; a
 * host-side counter for launch accounting. */
uint64_t md_launch_count(void);

/* Number of device memsets and device-to-device copies this library has
 * enqueued in this process so far (status words, arrival words, tables it
 * zeroes before accumulating); counted apart from the kernels. */
uint64_t md_memset_count(void);

/*
 * md_route_topk -- router top-k selection and gate weights.
 * "Expert Coupling in MoE Pretraining" (PicX summary), Background: each token
 * is routed to its top-k of E experts; Method 1: the routing probabilities
 * travel with the dispatched rows.
 *
 *   logits    float32 [T, E]   raw router logits (no NaN; -inf allowed; with
 *                              NaN the order is unspecified, but every token
 *                              still gets k distinct experts in [0, E))
 *   topk_idx  int32   [T, k]   out: experts by logit descending; equal
 *                              logits (-0.0 == +0.0) by lower expert index
 *   topk_w    float32 [T, k]   out: gate weights.  MD_GATE_TOPK_SOFTMAX:
 *                              softmax over the k selected logits;
 *                              MD_GATE_FULL_SOFTMAX: softmax over all E,
 *                              read at the selected experts.  Computed in
 *                              double from exact logit differences, rounded
 *                              to float once.
 *   Limits: 1 <= k <= min(E, 32), E <= 1024, T >= 0.
 */
int md_route_topk(const float *logits, int64_t T, int E, int k, int gate_mode,
                  int32_t *topk_idx, float *topk_w, void *stream);

/*
 * md_dispatch_layout -- rows, positions and the rank-by-rank send matrix.
 * "DODOCO: MoE AlltoAll Traffic Matrices on Real Text", send_matrices.csv and
 * Reading the counts: send_counts[s][d] counts what source rank s sends to
 * rank d; conventional counts are token-expert assignments (a row sums to
 * T/R x k); combine returns the transposed volumes.
 * "Expert Coupling in MoE Pretraining", Method 1: the deduplicating
 * dispatcher sends one row per distinct (token, destination rank) pair.
 *
 *   topk_idx        int32 [T, k]   experts per token (from md_route_topk)
 *   expert_to_rank  int32 [E]      p[e] in [0, R), exactly E/R experts per rank
 *   mode            MD_CONV or MD_DEDUP
 * Outputs:
 *   assign_row      int32 [T, k]   conventional row of (t, j): rows ordered by
 *                                  (p[e], e, t), e = topk_idx[t][j].  This is
 *                                  the expert-grouped order of the expert
 *                                  outputs md_combine reads, in both modes.
 *   row_of_slot     int32 [T, k]   row of (t, j) in this mode's layout; in
 *                                  MD_DEDUP rows are ordered by (d, t) and all
 *                                  slots of t on rank d share one row.
 *   row_token       int32 [T*k]    token of each row (first n_rows valid)
 *   row_mask        uint32 [T*k]   bit j set: the row carries slot j of its token
 *   send_counts     int32 [R, R]   rows from source rank s to rank d
 *   expert_counts   int32 [E]      tokens selecting expert e
 *   expert_offsets  int32 [E+1]    first conventional row of expert e; [E] = T*k
 *   rank_offsets    int32 [R+1]    first row of rank d in this mode; [R] = n_rows
 *   n_rows          int32 [1]      rows in this mode (T*k for MD_CONV)
 *   workspace       >= md_dispatch_layout_workspace_size(...) bytes, 256-B
 *                   aligned; contents on entry do not matter: the call clears
 *                   its arrival words on `stream` before the kernel (one 1 KiB
 *                   memset) and writes every count before reading it.  The
 *                   size does not grow with T (at most about 1.2 MiB, at
 *                   E=1024, R=64).
 *   One cooperative launch: all its CTAs (at most one per SM) must be
 *   resident at once, and every CTA waits for the others' counts with a
 *   bounded wait (MD_ERR_TIMEOUT in dev_status if it runs out; the outputs
 *   are then not written).  If the cooperative launch is refused (other work
 *   holds SMs), the call runs the same kernel split in two ordinary launches,
 *   counts then ranks, with identical results (md_set_layout_path).  Safe in
 *   CUDA graph capture: the graph records the clear of the arrival words
 *   with the kernel (a launch refused during capture ends the capture).
 *   Limits: T % R == 0, E % R == 0, 1 <= k <= min(E, 32), E <= 1024,
 *   R <= 64, T*k < 2^31.
 */
size_t md_dispatch_layout_workspace_size(int64_t T, int E, int k, int R, int mode);

int md_dispatch_layout(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                       const int32_t *expert_to_rank, int mode,
                       int32_t *row_of_slot, int32_t *assign_row,
                       int32_t *row_token, uint32_t *row_mask,
                       int32_t *send_counts, int32_t *expert_counts,
                       int32_t *expert_offsets, int32_t *rank_offsets, int32_t *n_rows,
                       void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, void *stream);

/*
 * md_dispatch_layout_noalloc -- md_dispatch_layout without a caller workspace.
 * No counterpart in the source pages: this is a calling convenience, not a
 * step of the method.  Some callers cannot allocate device memory at all --
 * for example a plug-in running inside a host framework that owns every byte
 * of GPU memory through its own pool, or a process that has handed all free
 * HBM to a caching allocator -- so they cannot size and cudaMalloc the
 * workspace md_dispatch_layout needs.  This entry point takes the same
 * arguments minus the workspace and allocates nothing: its scratch is a
 * fixed array of MD_NOALLOC_LAYOUT_SCRATCH_BYTES (4 MiB) compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  The caller still passes all inputs and outputs.
 *   - Every shape within md_dispatch_layout's limits fits: the workspace
 *     does not grow with T and is at most about 1.2 MiB.
 *   - The first call on each device looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; nothing in it has to start at zero.  Calls that
 *     overlap on the GPU (other streams, other threads) race on it and must
 *     be serialised by the caller.
 *   - Results are identical to md_dispatch_layout's.
 */
#define MD_NOALLOC_LAYOUT_SCRATCH_BYTES ((size_t)4 << 20)

size_t md_dispatch_layout_noalloc_max_scratch(void);

int md_dispatch_layout_noalloc(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                               const int32_t *expert_to_rank, int mode,
                               int32_t *row_of_slot, int32_t *assign_row,
                               int32_t *row_token, uint32_t *row_mask,
                               int32_t *send_counts, int32_t *expert_counts,
                               int32_t *expert_offsets, int32_t *rank_offsets, int32_t *n_rows,
                               int32_t *dev_status, void *stream);

/*
 * md_dispatch_permute -- build the dispatch buffer: out[row] = x[token(row)]
 * bit for bit.  "DODOCO ...", Reading the counts: the payload of a count is
 * hidden_size x bytes per element (bf16 here).
 * Token-major scatter: each x row is read once and written to every distinct
 * row named in row_of_slot[t][*] (slots sharing a row are written once).
 *
 *   x            bf16  [T, H]
 *   row_of_slot  int32 [T, k]   from md_dispatch_layout (either mode)
 *   out          bf16  [out_rows, H]; rows nobody names are left untouched
 *   A row index outside [0, out_rows) is skipped and reported (MD_ERR_DATA).
 */
int md_dispatch_permute(const void *x, int64_t T, int H, int k,
                        const int32_t *row_of_slot, int64_t out_rows, void *out,
                        int32_t *dev_status, void *stream);

/*
 * md_set_permute_path -- which kernel md_dispatch_permute runs (for tests and
 * tuning; the result is the same bits either way).
 *   MD_PERMUTE_AUTO    by shape (default): bulk copies through shared memory
 *                      for rows of at least 1 KiB when k > 4 and the call has
 *                      at least 8 row pieces of 4 KiB per warp of its grid;
 *                      16-byte vector loads and stores otherwise
 *   MD_PERMUTE_BULK    bulk copies whenever rows are at least 1 KiB
 *   MD_PERMUTE_VECTOR  16-byte vectors always
 * Process-wide; MD_ERR_ARG for another value.  Set it only while no
 * md_dispatch_permute call is being enqueued.
 */
#define MD_PERMUTE_AUTO 0
#define MD_PERMUTE_BULK 1
#define MD_PERMUTE_VECTOR 2

int md_set_permute_path(int path);

/*
 * md_set_layout_path -- the launch form of md_dispatch_layout (for tests and
 * for GPUs shared with other work; the results are the same either way).
 *   MD_LAYOUT_AUTO         one cooperative launch; if it is refused, the
 *                          split form (default)
 *   MD_LAYOUT_COOPERATIVE  one cooperative launch; MD_ERR_CUDA if refused
 *   MD_LAYOUT_SPLIT        always two launches: every CTA's counts, then the
 *                          ranks; no CTA waits on another
 * Process-wide; MD_ERR_ARG for another value.  Set it only while no
 * md_dispatch_layout call is being enqueued.
 */
#define MD_LAYOUT_AUTO 0
#define MD_LAYOUT_COOPERATIVE 1
#define MD_LAYOUT_SPLIT 2

int md_set_layout_path(int path);

/*
 * md_dedup_expand -- receiver-side expand of deduplicated rows.
 * "Expert Coupling ...", Method 1 (Deduplicating Dispatcher): a rank receives
 * one row per (token, rank) carrying all of the token's experts on that rank;
 * every selected expert then gets its own copy of the row, in the
 * conventional expert-grouped order (p[e], e, t) a grouped GEMM consumes.
 *
 *   wire         bf16  [n_wire, H]   dedup dispatch buffer (md_dispatch_permute
 *                                    with a MD_DEDUP layout)
 *   row_of_slot  int32 [T, k]        dedup row of each slot   } both from one
 *   assign_row   int32 [T, k]        conventional row of each } MD_DEDUP layout
 *   out          bf16  [out_rows, H] out[assign_row[t][j]] = wire[row_of_slot[t][j]]
 *                                    bit for bit; out_rows >= T*k for a full layout
 *   wire and out 16-byte aligned, H % 8 == 0.  A slot whose source or
 *   destination row is out of range is skipped and reported (MD_ERR_DATA).
 *   The result equals md_dispatch_permute with the conventional layout.
 */
int md_dedup_expand(const void *wire, int64_t n_wire, int H, const int32_t *row_of_slot,
                    const int32_t *assign_row, int64_t T, int k, int64_t out_rows, void *out,
                    int32_t *dev_status, void *stream);

/*
 * md_combine -- gate-weighted combine of the expert outputs.
 * "DODOCO ...", send_matrices.csv: combine, the second AlltoAll of each MoE
 * layer, returns the volumes of dispatch in reverse.  "Expert Coupling ...",
 * The Communication Bottleneck: dispatch and combine per MoE layer.
 *
 *   y            bf16  [y_rows, H]  expert outputs, row assign_row[t][j] holds
 *                                   expert topk_idx[t][j]'s output for token t
 *   assign_row, topk_idx int32 [T, k];  topk_w float32 [T, k]
 *   MD_COMBINE_FUSED: out[t] = bf16( sum over t's slots by ascending expert
 *                     of w * y, fp32 fused multiply-add from +0.0f ).
 *   MD_COMBINE_WIRE:  with row_of_slot from an MD_DEDUP layout: for each wire
 *                     row of t (ascending, i.e. ascending destination rank)
 *                     z[row] = bf16( same sum over the slots on that row );
 *                     out[t] = bf16( fp32 sum of the z rows in that order ).
 *                     z is bf16 [z_rows, H] (the return rows of the wire).
 *   out          bf16 [T, H]
 *   Row indices outside y_rows / z_rows are skipped and reported.
 */
int md_combine(const void *y, int64_t y_rows, const int32_t *assign_row,
               const int32_t *topk_idx, const float *topk_w, int64_t T, int k, int H,
               int combine_mode, const int32_t *row_of_slot, int64_t z_rows, void *z,
               void *out, int32_t *dev_status, void *stream);

/*
 * md_coselect_stats -- within-layer co-selection and cross-layer counts.
 * "Expert Coupling ...", Correlated Placement: W[e, e'] counts tokens
 * selecting both e and e' (diagonal: tokens selecting e); Cross-layer
 * correlation: experts chosen at layer l predict those at layer l+1.
 *
 *   idx_l     int32 [>= T_fit, k]  layer-l top-k
 *   idx_next  int32 [>= T_fit, k]  layer-l+1 top-k; may be NULL when C is NULL
 *             or T_fit is 0 (else MD_ERR_ARG)
 *   W         uint32 [E, E] or NULL: W[e][e'] += #{t < T_fit : e, e' in S_l(t)}
 *   C         uint32 [E, E] or NULL: C[e][e'] += #{(t,i,j) : S_l(t)_i = e,
 *                                                     S_l+1(t)_j = e'}
 *   accumulate  0: each table given is cleared first (T_fit = 0 leaves it
 *               zero); 1: counts are added.  At least one of W, C.
 *   Limits: E <= 1024, k <= 32.
 */
int md_coselect_stats(const int32_t *idx_l, const int32_t *idx_next, int64_t T_fit, int E,
                      int k, uint32_t *W, uint32_t *C, int accumulate, int32_t *dev_status,
                      void *stream);

/*
 * md_coselect_pair_stats -- pair counts for the pair-based shuffle predictor.
 * "Expert Coupling ...", Method 2 (Token Shuffling), Prediction: the next
 * layer is predicted from the experts of the two preceding layers.  Every
 * (a, b, e') triple of a token is counted, as C counts every (b, e') pair:
 *
 *   idx_prev, idx_l, idx_next  int32 [>= T_fit, k]  layers l-1, l, l+1
 *   C2  uint32 [E, E, E]: C2[a][b][e'] += #{(t,i,j,m) : S_l-1(t)_i = a,
 *                                 S_l(t)_j = b, S_l+1(t)_m = e'}, t < T_fit
 *   accumulate  0: C2 is cleared first; 1: counts are added.
 *   Limits: E <= MD_MAX_PAIR_EXPERTS (the table has E^3 entries), k <= 32.
 */
int md_coselect_pair_stats(const int32_t *idx_prev, const int32_t *idx_l, const int32_t *idx_next,
                           int64_t T_fit, int E, int k, uint32_t *C2, int accumulate,
                           int32_t *dev_status, void *stream);

/*
 * md_place_correlated -- correlated expert placement on the GPU.
 * "Expert Coupling ...", Correlated Placement: a Kernighan-Lin-style local
 * search from contiguous placement swaps experts between GPUs to maximise
 * the sum of W over co-located pairs; every GPU holds exactly E/EP experts.
 *
 *   W               uint32 [E, E], symmetric (from md_coselect_stats)
 *   seed_mode       MD_SEED_CONTIGUOUS or MD_SEED_GREEDY_PAIRS (pairs with
 *                   W > 0 by weight: both unplaced -> the rank with most free
 *                   slots if >= 2; one placed -> join it if room; leftovers
 *                   ascending into the lowest rank with room)
 *   refine          non-zero: repeat the best single swap (largest gain,
 *                   lowest expert pair on ties) while it gains, at most E*E
 *   expert_to_rank  int32 [E] out
 *   Limits: E % R == 0, E <= 1024, R <= 64.
 */
size_t md_place_correlated_workspace_size(int E, int R);

int md_place_correlated(const uint32_t *W, int E, int R, int seed_mode, int refine,
                        int32_t *expert_to_rank, void *workspace, size_t workspace_bytes,
                        int32_t *dev_status, void *stream);

/*
 * md_place_two_level -- placement with a choice of refinement and, for
 * multi-node groups, two levels ("Expert Coupling ...", Correlated
 * Placement: first across nodes, then across the GPUs within each node).
 *
 *   nodes        >= 1, R % nodes == 0; nodes == 1 is one level
 *   seed_mode    as md_place_correlated, at both levels
 *   refine_mode  MD_REFINE_NONE, MD_REFINE_SWAPS (as md_place_correlated) or
 *                MD_REFINE_KL: Kernighan-Lin passes -- in a pass, repeatedly
 *                the best swap among experts not yet moved in the pass
 *                (gain of any sign, lowest (a, b) on ties) until none is left
 *                or E/2 moves; keep the shortest prefix with the largest
 *                positive total, undo the rest; repeat while positive (at
 *                most E passes)
 *   Level 1 places experts on nodes (E/nodes each); level 2 places each
 *   node's experts, in ascending id, on its R/nodes ranks with W restricted
 *   to them: expert_to_rank[e] = node * (R/nodes) + rank within the node.
 *   Limits: E % R == 0, E <= 1024, R <= 64.
 */
size_t md_place_two_level_workspace_size(int E, int R, int nodes);

int md_place_two_level(const uint32_t *W, int E, int R, int nodes, int seed_mode, int refine_mode,
                       int32_t *expert_to_rank, void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, void *stream);

/*
 * md_token_shuffle -- capacity-constrained token shuffle to predicted owners.
 * "Expert Coupling ...", Method 2 (Token Shuffling), Mechanism: predict each
 * token's owner rank at layer l+1; every rank owns exactly T/EP tokens, so
 * tokens are assigned in decreasing confidence to their most preferred rank
 * with capacity left.  Single-expert prediction: token t with layer-l top-1
 * expert e1 prefers p_next[argmax_e' C[e1][e']] (lowest e' on ties), then
 * the other ranks by sum_{e' on d} C[e1][e'] descending (lowest d on ties);
 * confidence = max / sum of C's row e1 (exact rational comparison; an empty
 * row has confidence 0 and prefers src(t), then ascending ranks).  Tokens
 * are visited by (confidence desc, t asc).
 *
 *   idx_l                int32 [T, k]  layer-l top-k (column 0 is the top-1)
 *   C                    uint32 [E, E] layer l -> l+1 counts
 *   expert_to_rank_next  int32 [E]     layer-l+1 placement
 *   pred_rank  int32 [T]  out: rank each token is assigned to
 *   perm       int32 [T]  out: new position of token t; rank d's tokens take
 *                         d*T/R .. (d+1)*T/R-1 in ascending t
 *   inv        int32 [T]  out: inv[perm[t]] = t
 *   Limits: T % R == 0, E <= 1024, R <= 64, T < 2^31.
 */
size_t md_token_shuffle_workspace_size(int64_t T, int E, int R);

int md_token_shuffle(const int32_t *idx_l, int k, const uint32_t *C,
                     const int32_t *expert_to_rank_next, int64_t T, int E, int R,
                     int32_t *pred_rank, int32_t *perm, int32_t *inv,
                     void *workspace, size_t workspace_bytes, int32_t *dev_status,
                     void *stream);

/*
 * md_token_shuffle_rounds -- md_token_shuffle with a rounds-based parallel
 * capacity assignment in place of the sequential visit.  Priorities and
 * preference lists are md_token_shuffle's.  In each round every unassigned
 * token proposes to the first rank of its list that was not full when the
 * round began, and each rank accepts its highest-priority proposers up to
 * its remaining capacity; rounds repeat until every token is placed (at most
 * R + 1).  The result can differ from the sequential visit: a token turned
 * away by a full rank competes for its next choice one round later.
 *
 *   rounds  int32 [1] device, out (may be NULL): rounds that placed a token
 *   other arguments as md_token_shuffle; the workspace is
 *   md_token_shuffle_rounds_workspace_size bytes.
 *   All ceil(T/1024) CTAs of the assignment must be resident at once
 *   (cooperative launch): larger T returns MD_ERR_UNSUPPORTED.  Its grid
 *   barriers are bounded waits (MD_ERR_TIMEOUT).
 */
size_t md_token_shuffle_rounds_workspace_size(int64_t T, int E, int R);

int md_token_shuffle_rounds(const int32_t *idx_l, int k, const uint32_t *C,
                            const int32_t *expert_to_rank_next, int64_t T, int E, int R,
                            int32_t *pred_rank, int32_t *perm, int32_t *inv, int32_t *rounds,
                            void *workspace, size_t workspace_bytes, int32_t *dev_status,
                            void *stream);

/*
 * md_token_shuffle_pair -- md_token_shuffle with the pair-based prediction
 * and its single-expert fallback ("Expert Coupling ...", Method 2,
 * Prediction: a pair-based lookup over the two preceding layers, falling
 * back to single-expert prediction for sparse observations).  For token t
 * with top-1 experts a (layer l-1) and b (layer l), the prediction row is
 * C2[a][b] when its total is at least min_obs, else C[b]; preference order,
 * confidence, visit order (confidence desc, t asc) and the capacity rule are
 * those of md_token_shuffle applied to that row.
 *
 *   idx_prev   int32 [T, k]   layer-l-1 top-k (column 0 is the top-1)
 *   idx_l      int32 [T, k]   layer-l top-k
 *   C          uint32 [E, E]  layer l -> l+1 counts (md_coselect_stats)
 *   C2         uint32 [E, E, E] pair counts (md_coselect_pair_stats)
 *   min_obs    >= 1
 *   use_pair   int32 [T] out (may be NULL): 1 where the pair row was used
 *   other arguments as md_token_shuffle.
 *   Limits: T % R == 0, E <= MD_MAX_PAIR_EXPERTS, R <= 64, T < 2^31; every
 *   row total used must be below 2^31 (else MD_ERR_UNSUPPORTED in dev_status).
 */
size_t md_token_shuffle_pair_workspace_size(int64_t T, int E, int R);

int md_token_shuffle_pair(const int32_t *idx_prev, const int32_t *idx_l, int k, const uint32_t *C,
                          const uint32_t *C2, const int32_t *expert_to_rank_next, int64_t T, int E,
                          int R, uint32_t min_obs, int32_t *pred_rank, int32_t *perm, int32_t *inv,
                          int32_t *use_pair, void *workspace, size_t workspace_bytes,
                          int32_t *dev_status, void *stream);

/*
 * md_gather_rows -- dst[i] = src[index[i]] for i < n_out, rows of row_bytes.
 * Moves tokens into (index = inv) or out of (index = perm) the shuffled order
 * of md_token_shuffle ("Expert Coupling ...", Method 2: the all-gather
 * restores canonical order).  row_bytes must be a multiple of 4; src and dst
 * 16-byte aligned when row_bytes is a multiple of 16.  An index outside
 * [0, src_rows) leaves its row untouched and is reported (MD_ERR_DATA).
 */
int md_gather_rows(const void *src, int64_t src_rows, int64_t row_bytes, const int32_t *index,
                   int64_t n_out, void *dst, int32_t *dev_status, void *stream);

/*
 * Expert-parallel exchange between real ranks (one process per GPU).
 * "Expert Coupling ...", The Communication Bottleneck: dispatch and combine
 * are the two all-to-alls of each MoE layer; Method 1: a dedup row carries
 * the token's expert IDs and routing probabilities for its rank.  "DODOCO
 * ...", send_matrices.csv: source s sends send_counts[s][d] rows to rank d,
 * and combine returns the transposed volumes.
 *
 * Each rank lays out its own T_r tokens with md_dispatch_layout (rows
 * ordered (d, t)); its send row is rank_offsets[d+1] - rank_offsets[d].
 * After an all-gather of the R rank_offsets (the caller's collective),
 * md_exchange_plan places this rank's block in every destination: rank d
 * receives source 0's rows, then source 1's, ...  For MD_DEDUP layouts that
 * is the (d, global token) order of a single-GPU layout of all tokens; for
 * MD_CONV the rows arrive by (source, expert, token), and the receiver
 * groups them by expert for its GEMM (md_dedup_expand or its own order).  The data kernels
 * write or read the other ranks' buffers through plain device pointers
 * (peer pointers over NVLink, e.g. from symmetric memory or IPC handles, or
 * local memory); the caller orders them against the peers (a barrier
 * before md_combine_exchange reads what the peers wrote).  No load or store
 * uses multicast.
 *
 * md_peer_rows: one rank's buffers as seen by this rank (pointers on the
 * device, the struct itself in host memory):
 *   rows      bf16 [rows_cap, H]: dispatch receive rows (md_dispatch_exchange
 *             writes them) or combine return rows (md_combine_exchange reads)
 *   token     int32 [rows_cap] or NULL: global token id of each received row
 *   slot_idx  int32 [rows_cap, k] or NULL: per slot of the token, its expert
 *             if this row carries it (its expert sits on that rank), else -1
 *   slot_w    float [rows_cap, k] or NULL: the carried slots' gates, else 0
 *   row_base  first row of this source's block in those buffers
 *             (md_exchange_plan's dst_row_base[d])
 *   rows_cap  rows the buffers hold; a row outside [0, rows_cap) is skipped
 *             and reported (MD_ERR_DATA)
 */
typedef struct md_peer_rows {
    void *rows;
    int32_t *token;
    int32_t *slot_idx;
    float *slot_w;
    int64_t row_base;
    int64_t rows_cap;
} md_peer_rows;

/*
 * md_exchange_plan -- host helper (no device work; HOST pointers).
 *   src_rank_offsets  int64 [R, R+1]: every source rank's rank_offsets from
 *                     md_dispatch_layout of its own tokens, gathered (row s =
 *                     source s); source s sends rank_offsets_s[d+1] -
 *                     rank_offsets_s[d] rows to rank d (its send-matrix row)
 *   me                this rank
 *   dst_row_base      int64 [R] out: first row of my block on rank d, the
 *                     rows all sources before me send to d
 *   recv_offsets      int64 [R+1] out: first row of source s's block in my
 *                     receive buffer; [R] = rows I receive
 *   MD_ERR_DATA for a row that does not start at 0 or decreases.
 */
int md_exchange_plan(const int64_t *src_rank_offsets, int R, int me, int64_t *dst_row_base,
                     int64_t *recv_offsets);

/*
 * md_dispatch_exchange -- the dispatch all-to-all as one kernel: every
 * distinct row of each local token (rows shared by slots on one rank, in
 * an MD_DEDUP layout, travel once) is written bit for bit into its
 * destination rank's buffer, at peers[d].row_base + (row - rank_offsets[d]),
 * with its metadata (global token id token_base + t, slot experts, gates).
 *   x               bf16 [T, H], this rank's tokens
 *   topk_idx, topk_w  int32 / float [T, k] (topk_w may be NULL: gates 0)
 *   expert_to_rank  int32 [E]
 *   row_of_slot, rank_offsets  this rank's md_dispatch_layout of its tokens
 *   peers           host array of R md_peer_rows (rows required)
 *   Limits as md_dispatch_layout; H % 8 == 0, 16-byte aligned rows,
 *   token_base + T <= INT32_MAX.
 */
int md_dispatch_exchange(const void *x, int64_t T, int H, int k, const int32_t *topk_idx,
                         const float *topk_w, const int32_t *expert_to_rank, int E, int R,
                         const int32_t *row_of_slot, const int32_t *rank_offsets,
                         int64_t token_base, const md_peer_rows *peers, int32_t *dev_status,
                         void *stream);

/*
 * md_combine_partials -- on a receiving rank, the row that returns for each
 * received row i: z[i] = bf16(sum over the slots j it carries, in ascending
 * expert id, of slot_w[i][j] * y[y_row[i][j]]), fp32 fused multiply-add
 * from +0.0f (the first stage of MD_COMBINE_WIRE).
 *   y          bf16 [y_rows, H]: this rank's expert outputs
 *   y_row      int32 [n, k]: row of y holding slot j's expert output, or -1
 *              for a slot this row does not carry
 *   slot_idx, slot_w  int32 / float [n, k] as received
 *   z          bf16 [n, H] out
 */
int md_combine_partials(const void *y, int64_t y_rows, const int32_t *y_row,
                        const int32_t *slot_idx, const float *slot_w, int64_t n, int k, int H,
                        void *z, int32_t *dev_status, void *stream);

/*
 * md_combine_exchange -- the combine all-to-all as one kernel: for each local
 * token, the return rows of its ranks are read from the peers' buffers
 * (peers[d].rows at the same rows md_dispatch_exchange wrote) and
 * out[t] = bf16(fp32 sum of them in ascending rank) (the second stage of
 * MD_COMBINE_WIRE).  With an MD_DEDUP layout a token has one row per rank.
 *   out  bf16 [T, H]; other arguments as md_dispatch_exchange.
 */
int md_combine_exchange(const md_peer_rows *peers, int64_t T, int H, int k, const int32_t *topk_idx,
                        const int32_t *expert_to_rank, int E, int R, const int32_t *row_of_slot,
                        const int32_t *rank_offsets, void *out, int32_t *dev_status, void *stream);

/*
 * Routing statistics ("Expert Coupling ...").
 *
 * md_rank_stats -- Table I (Offline Placement and Prediction Statistics):
 *   hist  int64 [k+1] device, out: hist[D] = tokens whose k experts sit on
 *         exactly D distinct ranks under expert_to_rank.  "Same GPU" =
 *         hist[1] / T, "GPUs" = sum D hist[D] / T, "Dedup" = 1 - GPUs / k.
 *   An expert or rank out of range is reported (MD_ERR_DATA).
 *
 * md_successor_share -- Cross-layer correlation: with C (md_coselect_stats,
 *   layers l, l+1) and W (layer l) fitted on the same tokens, the share of
 *   expert e's tokens that select e' next is C[e][e'] / W[e][e].
 *   num uint32 [E] out: max_e' C[e][e'];  den uint32 [E] out: W[e][e].
 *
 * md_count_sums -- Correlation Formation and Stability: the Pearson
 *   correlation of two count tables x, y (uint32 [n]) follows from
 *   sums uint64 [10] device, out: (sx, sy, sxx, syy, sxy), each exact as a
 *   128-bit value in two words (low, high).  n < 2^31.
 */
int md_rank_stats(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                  const int32_t *expert_to_rank, int64_t *hist, int32_t *dev_status,
                  void *stream);

int md_successor_share(const uint32_t *C, const uint32_t *W, int E, uint32_t *num, uint32_t *den,
                       void *stream);

int md_count_sums(const uint32_t *x, const uint32_t *y, int64_t n, uint64_t *sums, void *stream);

/*
 * Host helpers that finish the statistics above (no device work; HOST
 * pointers; they may be called without a GPU).
 *
 * md_table1_row -- Table I columns ("Expert Coupling ...", Offline Placement
 *   and Prediction Statistics) from a rank histogram copied to the host:
 *   hist  int64 [k+1] host (md_rank_stats), T = sum of hist > 0
 *   out   double [3] host: "Same GPU" % = 100 hist[1] / T, "GPUs" = sum_D D
 *         hist[D] / T (mean distinct ranks per token), "Dedup" % = 100 (1 -
 *         GPUs / k).  MD_ERR_ARG for T == 0 or a negative entry.
 *
 * md_pearson_from_sums -- the Pearson correlation of two count tables of n
 *   entries (Correlation Formation and Stability) from md_count_sums' five
 *   exact sums copied to the host (uint64 [10]):
 *   r = (n sxy - sx sy) / sqrt((n sxx - sx^2)(n syy - sy^2)), the three
 *   differences exact in 128 bits, the quotient in long double.
 *   MD_ERR_DATA when a table has zero variance (r undefined) or the sums
 *   exceed what n 32-bit counts can give; 1 <= n < 2^31.
 */
int md_table1_row(const int64_t *hist, int k, double *out);

int md_pearson_from_sums(const uint64_t *sums, int64_t n, double *r);

/*
 * md_set_test_hooks -- fault injection for tests; not for production use.
 * Every bounded device-side wait gives up after a poll limit and reports
 * MD_ERR_TIMEOUT.  These hooks make such a wait run out on purpose, with no
 * fault: poll_limit > 0 replaces the default limits (md_route_topk then may
 * fall back to plain loads for a tile, with the same results); layout_skip_tile >= 0
 * makes that md_dispatch_layout CTA stamp no arrival word, so every CTA
 * waits for it in vain; expand_skip_unit >= 0 makes md_dedup_expand (bulk-copy
 * path) never fill that unit's shared-memory slot.  (0, -1, -1) restores the
 * defaults.  Process-wide; set them only while no other call is in flight.
 */
void md_set_test_hooks(long long poll_limit, int layout_skip_tile, long long expand_skip_unit);

#ifdef __cplusplus
}
#endif

#endif /* MOEDISPATCH_H */
