/*
 * dsa.h -- C ABI of libdsa: the DSA (DeepSeek-style Sparse Attention) hot path with
 * IndexShare for one NVIDIA B200 (sm_100a).
 *
 * The path has three steps and a driver:
 *   1. lightweight indexer score      I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s])
 *   2. per-query top-k select         the k best-scoring visible tokens
 *   3. sparse MLA attention           softmax attention over the selected compressed rows
 *   4. IndexShare group driver        1 x (1+2), then L x (3) with the same index list
 * Sources (page title, section): "GLM-5.2 1M architecture teardown" (clawlihai.cn),
 * Cut 1: DSA (an indexer coarse-screens 2048 of the history tokens; full attention runs
 * over those only; index_topk 2048, index_head_dim 128, index_n_heads 32), Cut 2:
 * IndexShare (the indexer sits in the first of every 4 layers and its top-k list is used
 * by all 4; index_topk_freq 4), Cut 3: MLA (a 512-wide compressed KV row per token);
 * "GLM-5.2 MTP IndexShare inference" (4sapi.ai), Indexer Share and its use in the MTP
 * layer (draft steps reuse the step-1 mask, so draft-token KV is never attended), KV
 * Share (the MTP layer reads the target model's cache); "Le contexte d'un million de
 * tokens" (glmmodel.cn), Attention sparse IndexShare and MTP avec IndexShare et KVShare.
 * The pages print no formula for the indexer score or the attention; the forms above
 * (and a 576-wide compressed row = 512 latent + 64 rope, value = first 512 entries) are
 * the readings this library implements.
 *
 * Conventions for every entry point
 *   - Tensors are caller-owned DEVICE pointers, dense row-major, in the layouts given.
 *     bf16 tensors are passed as uint16_t bit patterns.  bf16 tensors, the head weights,
 *     the output buffers and the workspace must be 16-byte aligned (the workspace
 *     256-byte); scores and index lists 4-byte.
 *   - Calls are asynchronous: work is enqueued on `stream` and the call returns.  The
 *     library allocates no memory and keeps no per-call state; scratch memory is the
 *     caller's `workspace` (size from dsa_workspace_size; dsa_group_forward also takes
 *     less, down to dsa_workspace_size_min).
 *   - Invalid arguments return an error before anything is enqueued.  DSA_ERR_CUDA
 *     reports a launch failure (cudaGetLastError after the launch).
 *   - Query t of a sequence sits at position q_pos0 + t and sees cached positions
 *     s <= q_pos0 + t, s < N (causal mask).  For decode, q_pos0 = N - 1.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misaligned pointer          */
    DSA_ERR_UNSUPPORTED = -2,  /* a shape the kernels do not implement                */
    DSA_ERR_WORKSPACE = -3,    /* workspace missing or too small (dsa_workspace_size;
                                  dsa_workspace_size_min for dsa_group_forward) */
    DSA_ERR_CUDA = -4,         /* a CUDA launch or runtime call failed                 */
    DSA_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up (see status word) */
    DSA_ERR_DEVICE = -6        /* a kernel recorded a device-side error                */
} dsa_status;

/* Fixed sizes of the path (GLM-5.2 configuration as quoted on the pages). */
#define DSA_INDEX_HEADS 32   /* index_n_heads                                          */
#define DSA_INDEX_DIM 128    /* index_head_dim                                         */
#define DSA_DQK 576          /* compressed row width: 512 latent + 64 rope             */
#define DSA_DV 512           /* value width: the first 512 entries of the row          */
#define DSA_MAX_TOPK 2048    /* index_topk                                             */
#define DSA_MAX_LAYERS 8     /* layers per dsa_group_forward call                      */

/* Human-readable name of a dsa_status value. */
const char *dsa_status_string(int status);

/*
 * The cudaError_t of the most recent call (on any thread) that returned DSA_ERR_CUDA, or 0
 * if none has; and the runtime's description of such a code.
 */
int dsa_last_cuda_error(void);
const char *dsa_cuda_error_string(int code);

/* Library version, major*10000 + minor*100 + patch. */
int dsa_version(void);

/*
 * Device-side error words.  The pipeline waits of the indexer and the attention kernels
 * are bounded: a wait that runs out records a nonzero code and the kernel returns early
 * (its outputs are then incomplete).  The top-k records a code when a selection invariant
 * fails (a row did not select exactly k positions), which would be a bug.
 *
 * dsa_check_device_status: synchronises `stream` (the work enqueued on it so far), reads
 * the error words and resets the ones that are set.  Returns DSA_ERR_TIMEOUT if a bounded
 * wait ran out, DSA_ERR_DEVICE if the top-k recorded a broken invariant, DSA_ERR_CUDA if
 * the stream itself reports a CUDA error, DSA_OK otherwise.  The words are per device and
 * shared by all streams: an error recorded by work on another stream shows here too.
 *
 * dsa_device_error: the same check after synchronising the whole device, also giving the
 * first nonzero code in *code (0 = none); clear != 0 resets the words.
 */
dsa_status dsa_check_device_status(cudaStream_t stream);
dsa_status dsa_device_error(int *code, int clear);

/*
 * Bytes of workspace needed by dsa_topk, dsa_sparse_attn and dsa_group_forward for these
 * sizes (one workspace serves all calls of that size).  B sequences, T queries per
 * sequence, N cached rows, k top-k, H attention heads, L layers per group.  The attention
 * part depends on the current device's SM count (how many CTAs share a query row), so
 * query it with the device that will run the calls current.  Returns 0 for invalid sizes.
 */
size_t dsa_workspace_size(int B, int T, int N, int k, int H, int L);

/*
 * The smallest workspace dsa_group_forward accepts for these sizes.  With fewer bytes than
 * dsa_workspace_size (the whole [B, T, N] score plane), a group call with T > 1 scores and
 * selects the query rows in chunks (of one sequence, a multiple of 8 rows, as many as the
 * workspace holds), each chunk's score plane reusing the same space -- the prefill's plane
 * is then never held whole (4096 x 131072 queries x keys: 2 GiB whole, 4.2 MB per 8-row
 * chunk).  The results are the same; a chunk whose plane fits L2 is read back from it.
 * The cost is time (measured on B200, 4096 queries, 4 layers: 14.9 ms with the whole
 * plane, 16.3 ms with 64 MiB of workspace, 25.1 ms with the minimum, 4.7 MiB).
 * Decode (T = 1) has no smaller form: the same as dsa_workspace_size.
 */
size_t dsa_workspace_size_min(int B, int T, int N, int k, int H, int L);

/*
 * Step 1 -- indexer score.
 *   q      [B, T, 32, 128]  bf16   indexer queries
 *   w      [B, T, 32]       f32    per-query head weights
 *   k      [B, N, 128]      bf16   index-key cache (one key per cached token)
 *   scores [B, T, N]        f32    out: I(t,s) for every visible s; entries with
 *                                  s > q_pos0 + t are unspecified
 * Products are bf16 x bf16, accumulated in f32 on the tensor cores.
 */
dsa_status dsa_index_score(const uint16_t *q, const float *w, const uint16_t *k,
                           int B, int T, int N, long long q_pos0, float *scores,
                           cudaStream_t stream);

/*
 * Step 1 over an FP8 index-key cache ("Le contexte d'un million de tokens", reinforcement
 * learning of the agent: an FP8 KV cache keeps memory within budget; the format is not
 * named there and E4M3 is taken: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits, subnormals, S.1111.111 = NaN).  Same layouts and output as dsa_index_score with
 * one byte per element of q and k, which halves the bytes of the key stream:
 *   q      [B, T, 32, 128]  E4M3   indexer queries
 *   w      [B, T, 32]       f32    per-query head weights
 *   k      [B, N, 128]      E4M3   index-key cache
 *   scores [B, T, N]        f32    out, as dsa_index_score
 * Products of E4M3 values are exact in f32; they are accumulated in f32 on the tensor
 * cores.
 */
dsa_status dsa_index_score_e4m3(const uint8_t *q, const float *w, const uint8_t *k,
                                int B, int T, int N, long long q_pos0, float *scores,
                                cudaStream_t stream);

/*
 * Step 2 -- top-k select.
 *   scores [B, T, N] f32 (only s <= q_pos0 + t is read)
 *   idx    [B, T, k] i32 out: the selected token positions in ascending order; when
 *                       fewer than k positions are visible all are kept and the rest
 *                       of the row is -1.
 * Order: higher score first; equal scores (-0 == +0) go to the lower token index; a NaN
 * ranks below every number.  Deterministic and bit-exact.  1 <= k <= 2048.
 */
dsa_status dsa_topk(const float *scores, int B, int T, int N, long long q_pos0, int k,
                    int32_t *idx, void *workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/*
 * Top-k select that allocates nothing -- for callers that cannot allocate device memory
 * when they run the select: an inference engine's plugin whose enqueue step must not
 * allocate (the engine owns every buffer), a serving loop held to a fixed memory plan, or
 * a latency-critical host thread that must not call cudaMalloc (it can synchronise the
 * device).  The pages have no counterpart of this entry point; it is the same select as
 * dsa_topk with the same bit-exact output, taking dsa_topk's arguments minus the
 * workspace.  Its scratch is a fixed DSA_NOALLOC_SCRATCH_BYTES array inside the library,
 * held on every GPU that loads the library until the process exits.
 *   - Shapes whose rows each fit one thread-block cluster on chip (decode shapes: rows of
 *     up to 262,144 visible positions, as many rows as the GPU runs clusters for at once)
 *     use no scratch.  The other shapes take the scan kernels, whose scratch must fit the
 *     array: at most 21 query rows (B*T) for N up to 1,048,576 (fewer for longer rows);
 *     beyond that the call returns DSA_ERR_WORKSPACE -- use dsa_topk.
 *   - The first call on a device looks up the array's device address (a runtime call,
 *     not an allocation).
 *   - All calls share the array and it keeps the last call's contents; the parts that
 *     must start at zero are cleared on `stream` by every call that uses them.  Calls that
 *     overlap on the GPU (unordered streams) race on the array and must not be issued.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (2u << 20)
dsa_status dsa_topk_noalloc(const float *scores, int B, int T, int N, long long q_pos0, int k,
                            int32_t *idx, cudaStream_t stream);

/*
 * Step 3 -- sparse MLA attention over the selected rows.
 *   q    [B, T, H, 576] bf16   attention queries (absorbed form)
 *   kv   [B, N, 576]    bf16   compressed cache; value = first 512 entries of a row
 *   idx  [B, T, k]      i32    selected rows (entries < 0 are skipped; all must be < N)
 *   out  [B, T, H, 512] f32    softmax_j(scale * q . kv[idx_j]) weighted sum of values;
 *                              zero when a row selects nothing
 * bf16 operands, f32 accumulation and softmax.  H in {16, 32, 48, 64}.
 * When few (row, layer) units are launched, each one's keys are split over up to 32 CTAs
 * (one per SM of the GPU in all) whose partial outputs meet in `workspace` (per split a
 * [64][512] f32 block and 64 (max, sum) pairs, 128.5 KB) and are merged by a second kernel
 * launched behind the first; dsa_workspace_size(B, T, N, k, H, 1) covers it.  Otherwise
 * (e.g. long prefill chunks) no workspace is read and it may be NULL.
 */
dsa_status dsa_sparse_attn(const uint16_t *q, const uint16_t *kv, const int32_t *idx,
                           int B, int T, int N, int H, int k, float scale, float *out,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Step 4 -- one IndexShare group (also one MTP draft step).
 *   iq, w, ik          indexer inputs as in dsa_index_score
 *   q[l], kv[l], out[l] for l < L: HOST arrays of L device pointers, one per layer, with
 *                       the layouts of dsa_sparse_attn
 *   compute_indices     1: run the indexer and top-k and write idx_shared;
 *                       0: use idx_shared as given (IndexShare layers 2..4 of a group,
 *                          MTP draft steps 2..7); iq, w, ik may then be NULL
 *   idx_shared [B,T,k]  the shared index list; never written when compute_indices = 0,
 *                       and read unchanged by all L layers
 *   workspace           dsa_workspace_size bytes, or fewer down to dsa_workspace_size_min
 *                       (the score plane in chunks of query rows, see there)
 * 1 <= L <= DSA_MAX_LAYERS.
 */
dsa_status dsa_group_forward(const uint16_t *iq, const float *w, const uint16_t *ik,
                             const uint16_t *const *q, const uint16_t *const *kv, int L,
                             int B, int T, int N, long long q_pos0, int H, int k, float scale,
                             int compute_indices, int32_t *idx_shared, float *const *out,
                             void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * A decode step over G IndexShare groups, micro-batched.  Per group: the indexer and the
 * top-k once, then the attention of L layers with the same index list (T = 1 query per
 * sequence at the newest cached position, q_pos0 = N - 1), exactly as dsa_group_forward
 * computes them.  The batch is split into two micro-batches -- sequences [0, ceil(B/2))
 * and the rest -- whose chains run on two streams: micro-batch 0 on `stream`, 1 on `side`
 * (a second stream of the caller; its work is joined back into `stream` before the call
 * returns, so the call completes on `stream` like any other).  Each micro-batch runs its
 * groups in order (group g+1's indexer after group g's attention, as in a model).  The
 * HBM-bound indexers of the two micro-batches take turns (each waits for the other's
 * previous one) on three quarters of the SMs, and each micro-batch's top-k and attention
 * run beside the other's indexer on the remaining quarter.  With B = 1, or with
 * side == stream, the groups run in order over the whole batch on `stream`, exactly like
 * one dsa_group_forward per group.  Which is faster depends on the row length (measured on
 * B200): with rows longer than a thread-block cluster's select holds (N > 262,144: the
 * long-row select, latency-bound) the two micro-batches hide it behind the other half's
 * indexer (1M contexts, B = 2: 871 against 1056 us per step of 8 groups; 512K: 654 against
 * 725 us); at 128K-256K the in-order step is faster (decode128k, B = 8: 97 against 138 us),
 * since the top-k and attention take nearly as long for half a batch as for all of it.  A decode step reads each selected row once,
 * so the attention gathers them under an L2 evict-first policy (dsa_group_forward keeps the
 * default policy: its caller may re-read the rows, as MTP draft steps do); the results are
 * the same either way.
 *   groups[g]   the group's tensors for all B sequences, in the layouts of
 *               dsa_group_forward with T = 1 (q, kv, out: L entries each)
 *   workspace   dsa_decode_workspace_size(B, N, k, H, L) bytes, 256-byte aligned
 * Uses events created once per device and host thread.
 */
#define DSA_INDEX_BF16 0 /* index_format: iq and ik hold bf16                          */
#define DSA_INDEX_E4M3 1 /* index_format: iq and ik hold E4M3 bytes (dsa_index_score_e4m3) */
typedef struct {
    const void *iq, *ik;     /* [B, 1, 32, 128] and [B, N, 128], element type index_format    */
    const float *w;          /* [B, 1, 32] f32                                                */
    const uint16_t *q[DSA_MAX_LAYERS];  /* [B, 1, H, 576] bf16 per layer                     */
    const uint16_t *kv[DSA_MAX_LAYERS]; /* [B, N, 576] bf16 per layer                        */
    int32_t *idx;                       /* [B, 1, k] out: the group's index list            */
    float *out[DSA_MAX_LAYERS];         /* [B, 1, H, 512] f32 per layer                     */
    int index_format;                   /* DSA_INDEX_BF16 or DSA_INDEX_E4M3                  */
} dsa_group_io;

size_t dsa_decode_workspace_size(int B, int N, int k, int H, int L);
dsa_status dsa_decode_step(const dsa_group_io *groups, int G, int L, int B, int N, int H, int k, float scale,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream, cudaStream_t side);

/*
 * Context-sharded decode ("Le contexte d'un million de tokens", Service efficace pour un
 * million de contextes: a long context is spread over several GPUs; the pages give no
 * algorithm).  Every GPU holds a contiguous range [offset, offset + N) of the cached tokens
 * of every sequence (index keys and compressed rows).  One step, with the exchanges done
 * by the caller (e.g. torch.distributed all-gathers over NCCL):
 *   1. dsa_index_score and dsa_topk on the shard (q_pos0 = the query's global position
 *      minus offset) give the shard's own top-k;
 *   2. dsa_shard_candidates turns it into (score, global position) candidates;
 *   3. the candidates of all shards are gathered, shard by shard in position order, and
 *      dsa_merge_candidates keeps the k best: the row's index list, identical to the
 *      unsharded top-k (a token in the row's top-k is in its shard's top-k);
 *   4. per layer, dsa_sparse_attn_shard attends over the selected rows the shard holds and
 *      returns the log-sum-exp of their logits beside the partial output;
 *   5. the partials of all shards are gathered and dsa_merge_partials combines them:
 *      out = sum_w exp(lse_w - LSE) out_w, LSE = ln sum_w exp(lse_w).
 */

/*
 * Step 3 on one shard.
 *   kv   [B, N, 576] bf16  the shard's compressed rows: global positions [offset, offset + N)
 *   idx  [B, T, k]   i32   global positions (entries < 0 or outside the shard are skipped)
 *   out  [B, T, H, 512] f32 out: softmax over the shard's selected rows only (0 if none)
 *   lse  [B, T, H]   f32   out: ln sum_j exp(scale * q . kv[j]) over them (-inf if none)
 * Otherwise as dsa_sparse_attn (workspace included).
 */
dsa_status dsa_sparse_attn_shard(const uint16_t *q, const uint16_t *kv, const int32_t *idx,
                                 int B, int T, int N, long long offset, int H, int k, float scale,
                                 float *out, float *lse, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream);

/*
 *   scores     [B, T, N] f32   the shard's indexer scores (as dsa_index_score wrote them)
 *   idx        [B, T, k] i32   the shard's top-k list (dsa_topk: shard-local positions)
 *   cand_score [B, T, k] f32   out: score of each entry (-inf for padding)
 *   cand_pos   [B, T, k] i32   out: its global position offset + idx (-1 for padding)
 */
dsa_status dsa_shard_candidates(const float *scores, const int32_t *idx, int B, int T, int N, int k,
                                long long offset, float *cand_score, int32_t *cand_pos,
                                cudaStream_t stream);

/*
 *   cand_score, cand_pos [W, B, T, kc]  the candidates of W shards, gathered shard-major
 *                          (as an all-gather leaves them), shards in position order, so
 *                          that the valid positions (>= 0) of a row increase from shard 0's
 *                          list to shard W-1's; W * kc <= 8 * 2048
 *   idx [B, T, k] i32 out: the k best by (score descending, position ascending; a NaN
 *                          ranks below every number), ascending, -1 padding when fewer
 *                          than k candidates are valid
 */
dsa_status dsa_merge_candidates(const float *cand_score, const int32_t *cand_pos, int W, int B,
                                int T, int kc, int k, int32_t *idx, cudaStream_t stream);

/*
 *   outs [W, B, T, H, 512] f32, lses [W, B, T, H] f32  the shards' partials
 *   out  [B, T, H, 512] f32 out: their log-sum-exp combination (0 where every lse is -inf)
 */
dsa_status dsa_merge_partials(const float *outs, const float *lses, int W, int B, int T, int H,
                              float *out, cudaStream_t stream);

/*
 * MTP verify step -- rejection sampling of the draft tokens ("GLM-5.2 MTP IndexShare
 * inference", Rejection Sampling: the acceptance rate is sum_v min(p_v, q_v); the MTP
 * pages verify the draft tokens in order and cut the sequence at the first rejection).
 *   p, q    [B, S, V] f32  target and draft probabilities of each draft position
 *                          (row b*S + j is position j of sequence b; values in [0, 1]);
 *                          V < 2^24
 *   draft   [B, S] i32     the draft tokens
 *   u, u2   [B, S] f32     uniform numbers in [0, 1): the accept test and the resample
 *   alpha   [B, S] f32 out the acceptance rate sum_v min(p_v, q_v)
 *   accept  [B, S] i32 out 1 iff u * q[x] < p[x] (float32), x the draft token
 *   token   [B, S] i32 out x when accepted, else a draw from max(0, p - q): integer
 *                          weights floor(max(0, p_v - q_v) * 2^40), target
 *                          floor(floor(u2 * 2^24) * sum / 2^24), the first token whose
 *                          inclusive prefix sum exceeds it (x when the residual is empty;
 *                          -1 for a draft token outside [0, V))
 *   accepted_len [B] i32 out the leading accepted positions of each sequence
 * Bit-exact decisions (accept, token, accepted_len); alpha within float32 summation error.
 */
dsa_status dsa_verify(const float *p, const float *q, const int32_t *draft, const float *u, const float *u2,
                      int B, int S, int V, float *alpha, int32_t *accept, int32_t *token, int32_t *accepted_len,
                      cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
