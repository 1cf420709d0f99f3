/*
 * pyr.h - C ABI of libpyr: hierarchical (pyramid) top-K key-block selection
 * and causal block-sparse attention for NVIDIA B200 (sm_100a).
 *
 * The problem, as the pages state it: queries, keys and values go in; each
 * query block gets a list of selected earlier key blocks; attention over
 * those blocks plus the query's own block comes out, with its log-sum-exp.
 *   - PISA abstract (peercurrent record): keys are pooled into a
 *     coarse-to-fine hierarchy of O(log N) levels; selection starts at the
 *     coarsest level and, level by level, applies LogSumExp scoring to a
 *     bounded candidate set, passing the survivors' children to the next
 *     finer level; the query-key score matrix is never materialised.
 *   - PHBA summary (paperlayer.ai), A.1.2 "Routing metadata kernels": block
 *     centroids average the block's key rows in fp32; routes go only to
 *     strictly preceding blocks; unavailable route slots hold -1.
 *   - PHBA summary, 3.1 "Top-K block routing" and A.1.3 "Query-tile fused
 *     sparse forward kernel": the current block is always attended with local
 *     causal attention; the forward pass keeps FlashAttention-style online
 *     softmax accumulators and writes the output and the log-sum-exp.
 *
 * Conventions shared by every entry point
 *   Layouts (row-major, contiguous, every base pointer 16-byte aligned):
 *     Q, O  [B][Hq][Nq][d]     K, V  [B][Hkv][N][d]
 *     pyr   [B][Hkv][P][2][d] bf16, level-major (level 0 first; node m of
 *           level l covers key blocks [m 2^l, min((m+1) 2^l, nb))). Each node
 *           mean x is stored as the unevaluated pair hi = RN_bf16(x),
 *           lo = RN_bf16(x - hi) (row [hi | lo]); x = hi + lo to 2^-17
 *           relative. This is the operand format of the tensor-core scoring.
 *     idx   [B][Hkv][nqb][topk] int32; gap [B][Hkv][nqb] fp32
 *     lse   [B][Hq][Nq] fp32 (natural log)
 *   Query row t sits at position q_offset + t. Key block j holds positions
 *   [j b, min((j+1) b, N)); query block i holds the query rows whose
 *   positions lie in [i b, (i+1) b). nb = ceil(N / b); nqb counts the query
 *   blocks that hold at least one query row. Selection is shared by the
 *   G = Hq / Hkv query heads of a kv head (grouped-query attention).
 *   Supported: d in {64, 128}; b in {16, 32, 64, 128}; dtype PYR_F32 or
 *   PYR_BF16 (Q, K, V and O share it); either decode (Nq == 1, any
 *   q_offset < N) or block-aligned prefill (q_offset % b == 0 and
 *   q_offset + Nq <= N); 1 <= topk <= cap <= 128, cap even; N % b may be
 *   non-zero (a ragged last block).
 *   Ownership: the caller allocates and owns every buffer; the library
 *   allocates nothing, keeps no state between calls beyond cached kernel
 *   attributes (and the copy streams of bsa_forward_host and the workspace
 *   array of bsa_backward_noalloc), and never frees caller memory.
 *   Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream). Calls only enqueue work and return; results are ready
 *   once the stream has been synchronised.
 *   Errors: the return value is the host-side status (PYR_OK, PYR_EINVAL,
 *   PYR_EUNSUPPORTED, PYR_ECUDA). Errors that only the device can see go to
 *   *dev_status when dev_status is non-NULL: a kernel stores its code there
 *   only if the word still holds PYR_OK, so the caller zeroes it before the
 *   calls and reads it after synchronising. No entry point aborts, throws or
 *   prints.
 */
#ifndef PYR_H
#define PYR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility even when the library is built
 * with -fvisibility=hidden. */
#if defined(__GNUC__)
#define PYR_API __attribute__((visibility("default")))
#else
#define PYR_API
#endif

#define PYR_OK 0
#define PYR_EINVAL 1       /* a NULL or misaligned pointer, or an inconsistent shape */
#define PYR_EUNSUPPORTED 2 /* a shape or dtype the library has no kernel for */
#define PYR_ECUDA 3        /* the CUDA runtime refused a launch */
#define PYR_ETIMEOUT 4     /* device: a bounded wait ran out (kernel returned early) */
#define PYR_EBADIDX 5      /* device: idx held a block that is not strictly before its query block */

#define PYR_F32 0
#define PYR_BF16 1

typedef struct pyr_shape {
  int B;        /* batch */
  int Hq;       /* query heads */
  int Hkv;      /* key/value heads; Hq % Hkv == 0 */
  int N;        /* key/value length */
  int Nq;       /* query rows per head */
  int q_offset; /* position of query row 0 */
  int d;        /* head dimension */
  int b;        /* block size: keys per key block, positions per query block */
  int topk;     /* K: key blocks kept per query block (the diagonal block is extra) */
  int cap;      /* candidate cap per pyramid level */
  int dtype;    /* PYR_F32 or PYR_BF16 */
} pyr_shape;

/* Number of pyramid levels, L + 1 with L = ceil(log2 nb); 0 on a bad shape. */
PYR_API int pyr_num_levels(const pyr_shape* s);

/* Number of pyramid nodes per (batch, kv head), P = sum over levels of
 * ceil(nb / 2^l); 0 on a bad shape. pyr holds B * Hkv * P * 2 * d bf16
 * values (4 * B * Hkv * P * d bytes). */
PYR_API int64_t pyr_num_nodes(const pyr_shape* s);

/* Query blocks per (batch, kv head), nqb; 0 on a bad shape. */
PYR_API int64_t pyr_num_qblocks(const pyr_shape* s);

/* Elements of the pyr buffer: B * Hkv * P * 2 * d bf16 values (the (hi, lo)
 * pair of every node mean), which is as many bytes as B * Hkv * P * d fp32
 * means; 0 on a bad shape. */
PYR_API size_t pyr_pyramid_elems(const pyr_shape* s);

/*
 * pyr_build - the key pyramid (PISA abstract: pooling builds O(log N) levels;
 * PHBA A.1.2: a centroid is the fp32 average of the block's key rows).
 *   K   device, [B][Hkv][N][d] in s->dtype (read only).
 *   pyr device, [B][Hkv][P][2][d] bf16 pairs (written): node (l, m) holds
 *       the mean of all keys under it, accumulated in fp32 and stored as
 *       (hi, lo); level-major, level 0 first.
 * Reads K once. Returns PYR_OK or a host-side error; nothing is written on
 * error.
 */
PYR_API int pyr_build(const pyr_shape* s, const void* K, void* pyr, int* dev_status, void* stream);

/*
 * pyr_means - the fp32 node means of a pyramid: means[u][n][e] = hi + lo of
 * node n's pair, for a caller that wants the pyramid as plain fp32 centroids
 * (PHBA A.1.2) rather than the (hi, lo) storage the walk reads.
 *   pyr   device, as written by pyr_build / pyr_update for the same shape.
 *   means device, [B][Hkv][P][d] fp32 (written), 4-byte aligned.
 * Enqueued on the stream like the other calls; returns PYR_OK or a
 * host-side error (nothing is written on error).
 */
PYR_API int pyr_means(const pyr_shape* s, const void* pyr, float* means, int* dev_status, void* stream);

/*
 * pyr_update - bring a pyramid up to date after the keys at positions
 * >= from_pos (0 <= from_pos < N) were rewritten, with the shape unchanged;
 * for example a decode step that writes its new key into the last slot. Only
 * the nodes whose key range reaches such a position are recomputed (one node
 * per level for a single position), from K for level 0 and from the children
 * above; large rewrites (more than 32 blocks) fall back to a full rebuild.
 *   K   device, [B][Hkv][N][d] in s->dtype (read only).
 *   pyr device, as written by pyr_build for the same shape (updated in place).
 * A context that grows past its current block count changes the level sizes
 * and needs pyr_build.
 */
PYR_API int pyr_update(const pyr_shape* s, const void* K, void* pyr, int from_pos, int* dev_status, void* stream);

/*
 * pyr_select - coarse-to-fine LogSumExp top-K key-block selection (PISA
 * abstract; routes to strictly preceding blocks with -1 padding, PHBA A.1.2).
 * For query block i of (batch, kv head), the node score is
 *   S = ln sum_r exp(q_r . kbar / sqrt(d)) + ln n_valid,
 * r running over every query row of block i in the G heads of the group;
 * kbar and n_valid are the mean and token count of the node's part that lies
 * before block i (nodes that start at or after block i are never scored).
 * The walk starts at the finest level with at most `cap` nodes, with every
 * valid node of that level as a candidate; each level above 0 keeps the best
 * min(cap/2, #candidates) (ties to the lower node index) and passes their
 * valid children on; level 0 keeps the best min(topk, #candidates).
 *   Q   device, [B][Hq][Nq][d] in s->dtype.
 *   pyr device, as written by pyr_build.
 *   idx device, [B][Hkv][nqb][topk] int32 (written): the kept blocks in
 *       ascending order, then -1. The query's own block is never listed.
 *   gap device, [B][Hkv][nqb] fp32 or NULL (written): the smallest score
 *       margin between the last kept and the first dropped candidate over
 *       the scored levels (+inf if no level dropped one).
 * Scoring accumulates in fp32.
 */
PYR_API int pyr_select(const pyr_shape* s, const void* Q, const void* pyr, int32_t* idx, float* gap,
                       int* dev_status, void* stream);

/*
 * Options of pyr_select_ex: the selection variants the PHAROS page (Zensar,
 * "Four mechanisms powering PHAROS") proposes as augmentations of
 * hierarchical selection, and a trace of the walk. All off in a zeroed struct,
 * which gives pyr_select's plain walk.
 *   budget     depth-sounding budget allocation (DBA: token budgets differ
 *              across heads): device [B][Hkv] int32, the number of level-0
 *              blocks each (batch, kv head) keeps, clamped to [0, topk]; NULL:
 *              topk - fcf_extra for every unit. The page derives the budgets
 *              from attention-head entropy without a formula, so they are an
 *              input here.
 *   fcf_tau,   fog-gate confidence fallback (FCF: the budget grows when
 *   fcf_extra  confidence is low): the confidence is the smallest margin
 *              between the last kept and the first dropped candidate over the
 *              levels above 0 and at the level-0 budget boundary; when it is
 *              below fcf_tau, level 0 keeps min(budget + fcf_extra, topk)
 *              blocks. fcf_extra = 0: off. fcf_tau must not be NaN.
 *   rcg_lambda range-light cross-level guidance (RCG: coarse levels guide the
 *              finer ones): candidates rank by R = S + rcg_lambda * R(parent),
 *              R = S at the start level; margins and gap are taken on R.
 *              0: off. Must be finite.
 *   trace      device [B][Hkv][nqb][levels][width] int32 or NULL (written):
 *              for level l, row levels - 1 - l lists the nodes kept at that
 *              level (any order), then -1; levels = pyr_select_trace_levels,
 *              width = pyr_select_trace_width. It records the walk so that it
 *              can be checked (or explained) level by level.
 * With a variant on, s->topk is the width of an idx row (the most blocks any
 * row may keep); rows keep their kept blocks ascending, then -1.
 */
typedef struct pyr_select_opts {
  const int32_t* budget;
  float fcf_tau;
  int fcf_extra;
  float rcg_lambda;
  int32_t* trace;
} pyr_select_opts;

/* Levels of a selection trace: the walk's start level (the finest with at
 * most cap nodes) down to 0; 0 on a bad shape. */
PYR_API int pyr_select_trace_levels(const pyr_shape* s);

/* Entries per trace level: max(cap / 2, topk); 0 on a bad shape. */
PYR_API int pyr_select_trace_width(const pyr_shape* s);

/*
 * pyr_select_ex - pyr_select with the options above (opts may be NULL). The
 * gap output becomes the smallest margin of any decision the walk took: at
 * every level the margin at the boundary it used, and, when the fallback
 * could change the result, the distance between the confidence and fcf_tau.
 * PYR_EINVAL for a negative fcf_extra, a NaN fcf_tau, a NaN or infinite
 * rcg_lambda, or a budget or trace pointer that is not 4-byte aligned.
 */
PYR_API int pyr_select_ex(const pyr_shape* s, const void* Q, const void* pyr, const pyr_select_opts* opts,
                          int32_t* idx, float* gap, int* dev_status, void* stream);

/*
 * bsa_forward - causal block-sparse attention (PHBA 3.1, 3.3 and A.1.3:
 * routed blocks plus the current block, one online-softmax merge, output and
 * log-sum-exp; the N x N score matrix is never formed).
 * Row t (position p, query block i, kv head h = hq / G) attends to every key
 * of the blocks idx[b][h][i - i0][*] (entries < 0 skipped) and to the keys of
 * block i at positions <= p, with softmax scale 1/sqrt(d).
 *   Q, K, V device, in s->dtype. idx device, as written by pyr_select: the
 *           non-negative entries of a row must be strictly ascending and < i;
 *           an entry that breaks this is skipped and PYR_EBADIDX is reported
 *           in *dev_status (the -1 entries may appear anywhere).
 *   O   device, [B][Hq][Nq][d] in s->dtype (written).
 *   lse device, [B][Hq][Nq] fp32 or NULL (written).
 * bf16 inputs run on the tcgen05 tensor cores (bf16 operands, fp32
 * accumulation in tensor memory); fp32 inputs run in fp32 on the CUDA cores.
 */
PYR_API int bsa_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                float* lse, int* dev_status, void* stream);

/*
 * PHBA prefix-state branch (PHBA summary, 2.2 "Gated slot memory", 3.2
 * "Prefix-state construction", 3.3 "Online-softmax token-state attention",
 * A.1.1 "Chunkwise parallel prefix-state memory construction", A.1.3).
 * Per (batch, kv head), an M-slot key state and an M-slot value state follow
 * one slot-wise retention gate a and one write gate w (the summary prints no
 * formula; the reading taken is)
 *   SK[s] <- a_t[s] SK[s] + w_t[s] ks_t,   SV[s] <- a_t[s] SV[s] + w_t[s] v_t,
 * from zero at position 0; the prefix state of key block j is (SK, SV) after
 * the tokens at positions < j b (block 0's is zero and is never attended:
 * its causal prefix is empty).
 * Layouts: PK, PV [B][Hkv][nb][M][d] in s->dtype; gates A (retention) and W
 * (write) [B][Hkv][N][M] fp32; 1 <= M <= 256.
 */

/* Elements of PK (and of PV): B * Hkv * nb * M * d; 0 on a bad shape or M. */
PYR_API size_t phba_state_elems(const pyr_shape* s, int M);

/* Device workspace bytes phba_state_build needs; 0 on a bad shape or M. */
PYR_API size_t phba_state_workspace_bytes(const pyr_shape* s, int M);

/*
 * phba_state_build - the prefix states of every key block, computed
 * chunkwise as the summary describes (A.1.1): within each block, every
 * token's decay to the block end (the product of the later retentions; a
 * log-A sum on the general path, a direct product on the bf16, d = 128,
 * b = 64, M % 32 == 0 path) weights its write, and the block's writes
 * become one decay-weighted matrix product; only the block-boundary states
 * are carried from block to block. fp32 arithmetic. The bf16, d = 128,
 * b = 64, M % 32 == 0 path does not touch the workspace.
 *   Ks        device, [B][Hkv][N][d] in s->dtype: the state branch's keys (the
 *             pages use un-rotated keys here; pass K when there is no rotation).
 *   V         device, [B][Hkv][N][d] in s->dtype.
 *   A, W      device, [B][Hkv][N][M] fp32: retention in [0, 1], write gate.
 *   PK, PV    device, [B][Hkv][nb][M][d] in s->dtype (written).
 *   workspace device, 16-byte aligned, >= phba_state_workspace_bytes bytes,
 *             caller-owned, contents on return unspecified.
 * s->topk and s->cap are ignored. The whole sequence [0, N) is one sequence
 * (the recurrence starts from zero at position 0).
 */
PYR_API int phba_state_build(const pyr_shape* s, int M, const void* Ks, const void* V, const float* A,
                             const float* W, void* PK, void* PV, void* workspace, size_t workspace_bytes,
                             int* dev_status, void* stream);

/*
 * phba_forward - bsa_forward extended with the prefix states (PHBA 3.3, A.1.3:
 * one softmax over the exact tokens and the prefix-state slots). Row t of
 * query block i attends, besides the keys bsa_forward gives it, to the M slots
 * of the state before block i (if i >= 1) and of the state before each routed
 * block j >= 1, each slot scored as qs_t . PK[slot] / sqrt(d) and carrying
 * value PV[slot].
 *   Q, K, V, idx, O, lse, dev_status: as for bsa_forward.
 *   Qs     device, [B][Hq][Nq][d] in s->dtype, or NULL (Q): the query the state
 *          slots are scored with (the pages use the un-rotated query).
 *   M      slots per state (0: plain bsa_forward); PK, PV as phba_state_build
 *          writes them.
 * bf16 prefill with d = 128 and Qs NULL (or Q) and M a multiple of 64 runs on
 * the tcgen05 tensor cores; every other case on the CUDA cores in fp32.
 */
PYR_API int phba_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx,
                         const void* Qs, int M, const void* PK, const void* PV, void* O, float* lse,
                         int* dev_status, void* stream);

/*
 * dense_forward - plain causal attention over every key at position <= p
 * (the FlashAttention-style consumer the PHAROS and PHBA pages compare
 * against), for finding the context length at which selection pays off.
 * Arguments as bsa_forward without idx; s->topk and s->cap are ignored.
 */
PYR_API int dense_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, void* O, float* lse,
                  int* dev_status, void* stream);

/*
 * bsa_forward_host - the whole forward path (pyr_build, pyr_select and
 * bsa_forward) for inputs and outputs in host memory. The pages state the
 * problem with Q, K and V as inputs and O and the log-sum-exp as outputs
 * (PHBA summary, 3.1 and A.1.3); this entry point takes them where a caller
 * without device copies of them holds them.
 * The (batch, kv head) units are independent through all three steps, so
 * they stream through the device in chunks of `units_per_chunk` consecutive
 * units (0: chunks that shrink towards the end of the call, from a quarter of
 * the units with at most 96 MiB of inputs each down to 2, 1, 1, so that the
 * per-chunk costs stay small and the last, unhidden chunk is one unit):
 * chunk c is computed on `stream` while
 * chunk c + 1 is copied in and chunk c - 1's output copied out on two copy
 * streams the library keeps per device (made on the first call on a device,
 * held until the process exits). O and lse are bit-identical to the three
 * device calls over the whole batch.
 *   Q, K, V   host, layouts as above (read).
 *   O         host, [B][Hq][Nq][d] in s->dtype (written).
 *   lse       host, [B][Hq][Nq] fp32, or NULL (written).
 *   workspace device, 16-byte aligned, at least
 *             pyr_host_workspace_bytes(s, units_per_chunk, lse != NULL)
 *             bytes, caller-owned; its contents on return are unspecified.
 *   dev_status device word, or NULL, as for the other entry points.
 * Host buffers should be page-locked (cudaHostAlloc, cudaHostRegister) for
 * the copies to overlap the compute; pageable memory gives the same result
 * with the copies serialised by the CUDA runtime.
 * The call enqueues and returns: everything it enqueues, on any stream, ends
 * before work the caller enqueues on `stream` afterwards, so O and lse are
 * ready, and the workspace and the host buffers are free, once `stream` has
 * been synchronised; the host inputs must stay unchanged until then. Work on
 * `stream` before the call is ordered before it. Calls on one device are
 * enqueued one at a time (a lock); calls that share a workspace must be
 * ordered on one stream.
 * Returns the host-side status; PYR_EINVAL also for a workspace that is too
 * small or misaligned. After an error part of the output may be written.
 */
PYR_API int bsa_forward_host(const pyr_shape* s, const void* Q, const void* K, const void* V, void* O, float* lse,
                             int units_per_chunk, void* workspace, size_t workspace_bytes, int* dev_status,
                             void* stream);

/* Device workspace bytes that bsa_forward_host needs for this shape, chunk
 * size (0 = automatic) and lse output (with_lse != 0); 0 on a bad shape or a
 * negative chunk size. */
PYR_API size_t pyr_host_workspace_bytes(const pyr_shape* s, int units_per_chunk, int with_lse);

/*
 * bsa_route_invert - the routes in block-major form, for the backward pass
 * (PHBA summary, A.1.2 "Routing metadata kernels": count the assignments per
 * key block, prefix-sum the counts into contiguous ranges, scatter the query
 * ids into them; route indices carry no gradient).
 *   idx    device, [B][Hkv][nqb][topk] int32, as written by pyr_select.
 *   offset device, [B*Hkv][nb + 1] int32 (written): unit u's key block j owns
 *          rho[u][offset[u][j] .. offset[u][j+1]).
 *   rho    device, [B*Hkv][nqb * topk] int32 (written): in each range, the
 *          query blocks qb (row index of idx) whose routes list j, ascending;
 *          entries past offset[u][nb] are -1. The query's own (diagonal)
 *          block is never listed.
 * A route that is not strictly before its query block, or that repeats in
 * its row, is left out and PYR_EBADIDX is reported in *dev_status. The result
 * does not depend on thread timing (each range is sorted).
 */
PYR_API int bsa_route_invert(const pyr_shape* s, const int32_t* idx, int32_t* offset, int32_t* rho, int* dev_status,
                             void* stream);

/*
 * bsa_backward - gradients of causal block-sparse attention (PHBA summary,
 * A.1.4 "Sparse backward kernel": a block-major schedule walks, for every key
 * block, the query rows that attend it; scores and probabilities are
 * recomputed on chip from the saved log-sum-exp). With the routes held fixed
 * and L = sum over rows of dO_t . O_t:
 *   P_tk = exp(q_t . k_k / sqrt(d) - lse_t),  D_t = dO_t . O_t,
 *   dS_tk = P_tk (dO_t . v_k - D_t),
 *   dQ_t = sum_k dS_tk k_k / sqrt(d),  dK_k = sum_t dS_tk q_t / sqrt(d),
 *   dV_k = sum_t P_tk dO_t,
 * t running over the rows of all G heads of the key's kv head.
 *   Q, K, V, O, dO device, in s->dtype (O and lse as written by bsa_forward).
 *   lse    device, [B][Hq][Nq] fp32.
 *   idx    device, as given to bsa_forward.
 *   offset, rho device, as written by bsa_route_invert from the same idx.
 *   delta  device, [B][Hq][Nq] fp32 workspace (overwritten with D_t).
 *   dQ     device, [B][Hq][Nq][d] in s->dtype (written). Before the dQ
 *          kernel writes it, its memory also holds the work list of the dK/dV
 *          kernel (bf16, d = 128, b = 64, G = 1), so it must not overlap any
 *          other argument.
 *   dK, dV device, [B][Hkv][N][d] in s->dtype (written, zero where no row
 *          attends).
 * Supported: whole-sequence prefill (q_offset == 0 and Nq == N); other
 * shapes return PYR_EUNSUPPORTED. Accumulation is fp32.
 */
PYR_API int bsa_backward(const pyr_shape* s, const void* Q, const void* K, const void* V, const void* O,
                         const float* lse, const void* dO, const int32_t* idx, const int32_t* offset,
                         const int32_t* rho, float* delta, void* dQ, void* dK, void* dV, int* dev_status,
                         void* stream);

/*
 * bsa_backward_noalloc - bsa_backward for callers that cannot allocate device
 * memory: plugins whose host framework owns all device memory and hands out
 * only the tensors it knows about, and serving or real-time loops that must not
 * call cudaMalloc (it can synchronise the device and block on the allocator).
 * The paper has no counterpart: this is a deployment variant of bsa_backward,
 * not part of the method.
 * Arguments and results are those of bsa_backward without `delta`: the
 * per-row workspace lives in a fixed array in the library's own device memory
 * (16 MiB per GPU that loads the library, held until the process exits), so
 * the call allocates nothing.
 *   Limit: B * Hq * Nq <= 4194304 query rows; larger shapes return
 *   PYR_EUNSUPPORTED without launching anything.
 *   The first call on a device looks up the array's device address (with that
 *   device current) and caches it; make that first call before any stream
 *   capture on the device.
 *   Every call on a device shares the one array. The workspace is written in
 *   full before it is read, so nothing needs clearing between calls, but calls
 *   that overlap on the GPU (on different streams, or from several threads
 *   without ordering) race on it: order them on one stream.
 */
PYR_API int bsa_backward_noalloc(const pyr_shape* s, const void* Q, const void* K, const void* V, const void* O,
                                 const float* lse, const void* dO, const int32_t* idx, const int32_t* offset,
                                 const int32_t* rho, void* dQ, void* dK, void* dV, int* dev_status, void* stream);

/*
 * pyr_selftest_wait - exercise the bounded waits the kernels rely on: one
 * kernel waits on an mbarrier that nothing arrives on and must give up after
 * its limit (about a second), store PYR_ETIMEOUT in *dev_status (device, must
 * not be NULL; zeroed by the caller) and return, leaving the context usable.
 * Not part of the method: a failure-detection check for callers and tests.
 */
PYR_API int pyr_selftest_wait(int* dev_status, void* stream);

/* Static, NUL-terminated description of a status code. */
PYR_API const char* pyr_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* PYR_H */
