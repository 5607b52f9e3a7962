/*
 * ra.h -- C ABI of the B200 (sm_100a) ring-chunked attention and Ulysses
 * layout-transform library (libra_b200.so).
 *
 * Sources, cited by page title and section:
 *   [SP-QA]   "Как работает sequence parallelism в контексте LLM?" (Q&A page on
 *             sequence parallelism): section 2 "Базовый принцип: разрезание
 *             последовательности" (contiguous chunking), section 3 "Ring
 *             Attention — эффективная коммуникация" (the P-step ring), section 5
 *             "Практическая реализация: псевдокод ring attention" (per-chunk
 *             scores, online-softmax / log-sum-exp merge, final normalisation).
 *   [ULYSSES] "Метод контекстного параллелизма Ulysses" (post on Ulysses context
 *             parallelism): the all-to-all from [local_seqlen, global_heads,
 *             head_dim] to [global_seqlen, local_heads, head_dim] and back, and
 *             the GQA rule that KV heads are copied up to the CP-group size.
 *   [ACCEL-SP] "Paralelismo de secuencias en 🤗 accelerate", section "En qué se
 *             diferencia Ulysses SP de FSDP CP": Ulysses needs the head count
 *             divisible by the number of ranks; ring attention does not; section
 *             "Configuración del backend SP de ALST/Ulysses": position_ids and
 *             packed samples.
 *
 * The P "ranks" of the ring are virtual: P chunk partitions held in the memory
 * of one GPU. Nothing here communicates between devices.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer into memory the caller owns and
 *     keeps alive until the work queued on `stream` has finished.  The library
 *     allocates no device memory and keeps no reference after the call returns.
 *   - Arrays of chunk pointers (k_chunks, v_chunks) are HOST arrays of device
 *     pointers; they are read during the call only.
 *   - Every tensor is dense, row-major, in the element type named by its dtype
 *     argument, unless a stride argument says otherwise.  Every device pointer
 *     must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously; the return status covers argument
 *     validation and the launch only.  A kernel that gives up on a bounded
 *     internal wait records that in a per-device error word, which
 *     ra_sync_status() reads back.
 *   - On any status other than RA_OK nothing has been enqueued, except for
 *     RA_ERR_CUDA after a failed launch, and ra_last_error() returns a message
 *     describing the problem (thread-local, valid until the next call on the
 *     same thread).
 *   - Outputs must not alias inputs unless an entry point says so.
 */
#ifndef RA_B200_H
#define RA_B200_H

#if defined(__GNUC__)
#define RA_API __attribute__((visibility("default")))
#else
#define RA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RA_OK = 0,
    RA_ERR_INVALID = 1,      /* bad argument: null/misaligned pointer, bad size or divisibility */
    RA_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement (e.g. D not in {32,64,128}) */
    RA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed; see ra_last_error() */
    RA_ERR_TIMEOUT = 4       /* a kernel gave up on a bounded internal wait; outputs are undefined */
} ra_status;

typedef enum {
    RA_BF16 = 0,  /* bfloat16, 2 bytes */
    RA_FP32 = 1   /* IEEE binary32, 4 bytes */
} ra_dtype;

/*
 * ra_ring_attn_fwd -- exact attention of every query row against P K/V chunks,
 * computed chunk by chunk in ring order with an online-softmax (log-sum-exp)
 * merge after each chunk step.  [SP-QA] sections 2, 3 and 5.
 *
 * Sequence: global length L = P*Lc.  Virtual rank i owns the contiguous tokens
 * [i*Lc, (i+1)*Lc) ([SP-QA] section 2).  For the queries of rank i, chunk step s
 * (s = 0..P-1) attends to the K/V chunk j = (i - s) mod P ([SP-QA] section 3:
 * each rank passes its chunk to the next rank, so at step s it holds the chunk
 * of rank i-s), and merges the partial result into the running one by the
 * log-sum-exp rule of [SP-QA] section 5.
 *
 * Result, per batch b, query position t, query head h (kv head g = h/(H_q/H_kv)):
 *   s_j      = scale * sum_d q[b,t,h,d] * k[b,j,g,d]   for visible j
 *   lse      = log(sum_j exp(s_j))                       (natural log)
 *   out[...] = sum_j exp(s_j - lse) * v[b,j,g,:]
 * Visible keys: all j < L, or with causal != 0 the keys j <= t (global
 * positions in rank order).  Chunk pairs whose keys are all invisible issue no
 * work.  Every query row sees at least one key.
 *
 * Arguments
 *   q          device, in_dtype, [B][P*Lc][H_q][D]; batch b starts at
 *              q + b*q_bstride elements (q_bstride >= P*Lc*H_q*D).
 *   k_chunks   host array of P device pointers; chunk j is [B][Lc][H_kv][D]
 *              in_dtype, batch b of chunk j starts at k_chunks[j] + b*kv_bstride
 *              elements (kv_bstride >= Lc*H_kv*D).
 *   v_chunks   as k_chunks, same kv_bstride.
 *   P          number of virtual ranks, 1 <= P <= RA_MAX_P.
 *   B, H_q, H_kv, Lc, D   sizes; H_q % H_kv == 0 (grouped-query attention).
 *   scale      multiplier of the raw scores (typically 1/sqrt(D)).
 *   causal     0 or 1.
 *   in_dtype   RA_BF16 (tcgen05 tensor-core path; D in {64,128}) or RA_FP32
 *              (CUDA-core fp32 path; D in {32,64,128}).
 *   out_dtype  RA_FP32 or RA_BF16 (BF16 only with in_dtype RA_BF16).
 *   out        device, out_dtype, dense [B][P*Lc][H_q][D] (normalised output).
 *   lse        device, fp32, dense [B][H_q][P*Lc], natural-log log-sum-exp.
 *   stream     cudaStream_t.
 * Errors: RA_ERR_INVALID for null or misaligned pointers, P < 1 or P > RA_MAX_P,
 *   B/H_q/H_kv/Lc < 1, H_q % H_kv != 0, strides below the dense size, causal
 *   not in {0,1}, out_dtype BF16 with fp32 input; RA_ERR_UNSUPPORTED for D
 *   outside the lists above.
 */
#define RA_MAX_P 64
RA_API ra_status ra_ring_attn_fwd(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           int P, int B, int H_q, int H_kv, int Lc, int D,
                           long long q_bstride, long long kv_bstride,
                           float scale, int causal, ra_dtype in_dtype, ra_dtype out_dtype,
                           void* out, float* lse, void* stream);

/*
 * ra_ring_attn_fwd_zigzag -- ra_ring_attn_fwd for shards in the zigzag layout.
 * [ULYSSES] names ZigZag beside the plain ring among the context-parallel
 * methods (introduction) without describing it; the layout taken here is the
 * load-balanced one for causal attention: the sequence of L = P*Lc tokens (Lc
 * even) is cut into 2P segments of Lc/2 tokens and rank i holds segment i
 * followed by segment 2P-1-i, so under a causal mask every rank has the same
 * work.  The ring schedule, the merge and the result formula are those of
 * ra_ring_attn_fwd; only the sequence position of each token changes:
 *   local token u of rank j's shard (row j*Lc + u of q and of out/lse, row u
 *   of chunk j) sits at position u < Lc/2 ? j*Lc/2 + u : (2P-1-j)*Lc/2 + u - Lc/2,
 * and with causal != 0 a key is visible to a query when its position is not
 * after the query's.  Without causal masking the result equals
 * ra_ring_attn_fwd's (positions then play no role).
 * Arguments, layout, ownership and errors: as ra_ring_attn_fwd, plus
 *   RA_ERR_INVALID when Lc is odd.
 */
RA_API ra_status ra_ring_attn_fwd_zigzag(const void* q, const void* const* k_chunks,
                                         const void* const* v_chunks, int P, int B, int H_q,
                                         int H_kv, int Lc, int D, long long q_bstride,
                                         long long kv_bstride, float scale, int causal,
                                         ra_dtype in_dtype, ra_dtype out_dtype, void* out,
                                         float* lse, void* stream);

/*
 * ra_ring_attn_fwd_packed -- causal ra_ring_attn_fwd over packed samples.
 * [ACCEL-SP] section "Configuración del backend SP de ALST/Ulysses": sequence
 * parallelism there is driven by position_ids rather than an attention mask,
 * and several samples may be combined into one sequence, attention staying
 * inside each.  The reading taken: the samples of a batch row are contiguous,
 * position_ids count 0, 1, 2, ... within each sample, and a sample starts where
 * position_ids is 0.  Query t of batch row b then sees exactly the keys
 * t - position_ids[b][t] .. t (its own sample, up to itself); the ring
 * schedule, the merge and the result formula are those of ra_ring_attn_fwd
 * (contiguous shards, causal).  Tiles and chunks holding no key a row block may
 * see issue no work, so short samples cost what their own attention costs.
 * Arguments, layout, ownership and errors: as ra_ring_attn_fwd (without
 * `causal`, which is implied), plus
 *   position_ids  device, int32, dense [B][P*Lc], 4-byte aligned; read only.
 *                 Ids that break the rule above are not detected: each query
 *                 t then sees the keys max(0, t - id) .. t.
 *   RA_ERR_INVALID when position_ids is null or misaligned.
 */
RA_API ra_status ra_ring_attn_fwd_packed(const void* q, const void* const* k_chunks,
                                         const void* const* v_chunks, const int* position_ids,
                                         int P, int B, int H_q, int H_kv, int Lc, int D,
                                         long long q_bstride, long long kv_bstride, float scale,
                                         ra_dtype in_dtype, ra_dtype out_dtype, void* out,
                                         float* lse, void* stream);

/*
 * ra_ring_attn_bwd -- the backward pass of ra_ring_attn_fwd (contiguous shards):
 * the gradients of out with respect to q, k and v given dout = dLoss/dout.
 * [SP-QA] trains with ring attention (the long-context training the pages
 * motivate); the pages print no gradient, so this is the derivative of the
 * forward's definition:
 *   P_ij  = exp(s_ij - lse_i)            (s as in ra_ring_attn_fwd; lse from it)
 *   Delta_i = sum_d dout[i][d] * out[i][d]
 *   dS_ij = P_ij * (dout_i . v_j - Delta_i)
 *   dq_i = scale * sum_j dS_ij k_j;  dk_j = scale * sum_i dS_ij q_i;  dv_j = sum_i P_ij dout_i
 * with i over the query rows (of every query head sharing the kv head) that see
 * key j.  Computed on the tensor cores: a row reduction for Delta (which also
 * zeroes dq), then one kernel with the key tile stationary that visits the query
 * tiles seeing its keys (causal tiles skipped), accumulates dk and dv, and adds
 * each tile pair's share of dq into dq in global memory (fp32 reduce-adds).
 * Reproducibility: dk and dv are the same bits on every call with the same
 * inputs; dq is the same up to the rounding of its fp32 sum, whose order of
 * additions across key tiles varies from call to call.  With
 * ra_set_bwd_deterministic(1) dq is computed instead by a second kernel with the
 * query tile stationary (every element summed in one fixed order and written
 * once), so that all three gradients are the same bits on every call.
 * Arguments
 *   q, k_chunks, v_chunks, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride,
 *   scale, causal   exactly as given to ra_ring_attn_fwd (bf16, D in {64,128}).
 *   out        device, bf16, dense [B][P*Lc][H_q][D]: the forward's output.
 *   lse        device, fp32, dense [B][H_q][P*Lc]: the forward's log-sum-exp.
 *   dout       device, bf16, dense [B][P*Lc][H_q][D].
 *   dq         device, fp32, dense [B][P*Lc][H_q][D] (written; its prior contents
 *              are never read).
 *   dk_chunks, dv_chunks  host arrays of P device pointers, chunk j fp32 dense
 *              [B][Lc][H_kv][D] (written).
 *   workspace  device, fp32, [B][H_q][P*Lc] scratch owned by the caller (holds
 *              Delta between the kernels; its contents on return are unspecified).
 *   stream     cudaStream_t.
 * Errors: as ra_ring_attn_fwd for the shared arguments; RA_ERR_INVALID for null
 *   or misaligned out, lse, dout, dq, workspace or gradient chunk pointers;
 *   RA_ERR_UNSUPPORTED for D outside {64, 128}.
 */
RA_API ra_status ra_ring_attn_bwd(const void* q, const void* const* k_chunks,
                                  const void* const* v_chunks, const void* out,
                                  const float* lse, const void* dout, int P, int B, int H_q,
                                  int H_kv, int Lc, int D, long long q_bstride,
                                  long long kv_bstride, float scale, int causal, float* dq,
                                  float* const* dk_chunks, float* const* dv_chunks,
                                  float* workspace, void* stream);

/*
 * ra_ring_attn_bwd_accumulate -- ra_ring_attn_bwd that adds this call's gradients into dq,
 * dk_chunks and dv_chunks instead of overwriting them.  It is the per-step call of a ring
 * backward across devices ([SP-QA] section 5, carried to the gradient): each step adds the
 * share of one K/V chunk, computed with the forward's FINAL out and lse (those of the whole
 * sequence), into the query chunk's dq and into the dk, dv accumulators that travel with
 * the K/V chunk; summed over the chunks, the shares are the gradients.
 * Arguments as ra_ring_attn_bwd, except: dq, dk_chunks, dv_chunks hold valid fp32 values on
 * entry (zeros, or earlier shares) and receive the sums.  With causal = 1 the call is one
 * chunk's own (diagonal) step; a wholly visible chunk is causal = 0.  out and lse are the
 * forward's results over the whole sequence for these query rows.
 * Reproducibility: as ra_ring_attn_bwd (dk, dv: fixed order; dq: the order of its fp32
 * additions across key tiles varies).
 * Errors: as ra_ring_attn_bwd.
 */
RA_API ra_status ra_ring_attn_bwd_accumulate(const void* q, const void* const* k_chunks,
                                             const void* const* v_chunks, const void* out,
                                             const float* lse, const void* dout, int P, int B,
                                             int H_q, int H_kv, int Lc, int D,
                                             long long q_bstride, long long kv_bstride,
                                             float scale, int causal, float* dq,
                                             float* const* dk_chunks, float* const* dv_chunks,
                                             float* workspace, void* stream);

/*
 * ra_ring_attn_bwd_zigzag -- ra_ring_attn_bwd for shards in the zigzag layout: the
 * gradients of ra_ring_attn_fwd_zigzag.  The same definition with every token at its
 * sequence position (the layout of ra_ring_attn_fwd_zigzag); dq, dk_chunks and
 * dv_chunks are in the same shard layout as q, k_chunks and v_chunks.
 * Arguments as ra_ring_attn_bwd.  Errors: as ra_ring_attn_bwd; RA_ERR_INVALID when Lc
 * is odd.
 */
RA_API ra_status ra_ring_attn_bwd_zigzag(const void* q, const void* const* k_chunks,
                                         const void* const* v_chunks, const void* out,
                                         const float* lse, const void* dout, int P, int B,
                                         int H_q, int H_kv, int Lc, int D, long long q_bstride,
                                         long long kv_bstride, float scale, int causal,
                                         float* dq, float* const* dk_chunks,
                                         float* const* dv_chunks, float* workspace, void* stream);

/*
 * ra_ring_attn_bwd_packed -- ra_ring_attn_bwd over packed samples: the gradients of
 * ra_ring_attn_fwd_packed (causal; query t of batch row b sees the keys
 * t - position_ids[b][t] .. t).  Every gradient is the sum over the pairs that the forward
 * attended, so each sample's gradients are those of its own causal attention.
 * position_ids: device, int32, [B][P*Lc] (the forward's).  Other arguments as
 * ra_ring_attn_bwd (causal is implied).  Errors: as ra_ring_attn_bwd; RA_ERR_INVALID when
 * position_ids is null or misaligned.
 */
RA_API ra_status ra_ring_attn_bwd_packed(const void* q, const void* const* k_chunks,
                                         const void* const* v_chunks, const int* position_ids,
                                         const void* out, const float* lse, const void* dout,
                                         int P, int B, int H_q, int H_kv, int Lc, int D,
                                         long long q_bstride, long long kv_bstride, float scale,
                                         float* dq, float* const* dk_chunks,
                                         float* const* dv_chunks, float* workspace, void* stream);

/*
 * ra_ring_attn_bwd_static -- ra_ring_attn_bwd without a workspace argument: the Delta
 * rows live in a fixed device array inside the library, so a call allocates no device
 * memory (no cudaMalloc, no cudaFree, no allocating library routine).  The pages have no
 * counterpart to this entry point; it is a deployment convenience around the backward.
 * Arguments and results are those of ra_ring_attn_bwd, minus workspace.
 * Limit: B * H_q * P * Lc <= RA_BWD_STATIC_MAX_ROWS (2^21 rows, an 8 MiB fp32 array per
 *   device); larger requests return RA_ERR_INVALID before anything is enqueued.
 * Set-up: every call looks the array's address up in the context current at the call
 *   (cudaGetSymbolAddress; nothing is cached, so after cudaDeviceReset or any other
 *   teardown and re-creation of the context the next call finds the array in the new
 *   context).  The first call in a context may load the library's device code and sets
 *   the kernels' shared-memory attributes; make that first call before any stream
 *   capture.
 * Concurrency: the array is shared by all calls on a device.  Calls that overlap in time
 *   (on different streams, or from host threads without ordering between them) race on
 *   it; calls ordered on one stream do not.  Nothing in it needs to start at zero.
 * Errors: those of ra_ring_attn_bwd; RA_ERR_INVALID when the size limit is exceeded;
 *   RA_ERR_CUDA if the array's address cannot be obtained in the current context.
 */
#define RA_BWD_STATIC_MAX_ROWS (1 << 21)
RA_API ra_status ra_ring_attn_bwd_static(const void* q, const void* const* k_chunks,
                                         const void* const* v_chunks, const void* out,
                                         const float* lse, const void* dout, int P, int B,
                                         int H_q, int H_kv, int Lc, int D,
                                         long long q_bstride, long long kv_bstride, float scale,
                                         int causal, float* dq, float* const* dk_chunks,
                                         float* const* dv_chunks, void* stream);

/*
 * ra_lse_merge -- merge two partial attention results over disjoint key sets
 * into one, in place into (o_a, lse_a).  [SP-QA] section 5 (the merge step of
 * the ring loop, read as the exact log-sum-exp combination):
 *   lse      = log(exp(lse_a) + exp(lse_b))
 *   o_a[...] = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b
 * A partial over no visible key is (o = anything finite, lse = -inf); merging
 * with it leaves the other side unchanged, and two such partials merge to
 * (0, -inf).
 *   o_a, o_b     device fp32, [B][L][H][D]  (o_a is read and overwritten)
 *   lse_a, lse_b device fp32, [B][H][L]     (lse_a is read and overwritten)
 * o_b/lse_b must not alias o_a/lse_a.  Errors: RA_ERR_INVALID for null or
 * misaligned pointers or sizes < 1; RA_ERR_UNSUPPORTED if D % 4 != 0.
 */
RA_API ra_status ra_lse_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b,
                       int B, int H, long long L, int D, void* stream);

/*
 * ra_ulysses_seq2head -- the Ulysses layout transform from sequence-sharded to
 * head-sharded activations, for all P virtual ranks at once.  [ULYSSES]: the
 * all-to-all that turns [local_seqlen, global_heads, head_dim] into
 * [global_seqlen, local_heads, head_dim]; with GQA the KV heads are first
 * copied up so that every rank gets one ([ULYSSES], [ACCEL-SP]).
 *
 *   in   device, dt, [P][B][Lc][H_in][D]   (rank s holds tokens s*Lc .. s*Lc+Lc-1)
 *   out  device, dt, [P][B][P*Lc][H_out/P][D]
 *   out[r][b][s*Lc+t][h'][:] = in[s][b][t][ ((r*H_out/P + h') * H_in) / H_out ][:]
 * Rank r receives the contiguous head block [r*H_out/P, (r+1)*H_out/P) of the
 * H_out (replicated) heads; replica j of the H_out heads is a copy of source
 * head floor(j*H_in/H_out) (repeat-interleave).  H_out == H_in is the plain
 * transform.  The copy is bit-exact.
 * Errors: RA_ERR_INVALID for null/misaligned pointers, sizes < 1,
 *   H_out % P != 0 (heads must divide among ranks), H_out % H_in != 0,
 *   D*sizeof(dt) % 16 != 0.
 */
RA_API ra_status ra_ulysses_seq2head(const void* in, void* out, int P, int B, int Lc,
                              int H_in, int H_out, int D, ra_dtype dt, void* stream);

/*
 * ra_ulysses_head2seq -- the inverse transform, after attention and before the
 * output projection ([ULYSSES]):
 *   in   device, dt, [P][B][P*Lc][H/P][D]
 *   out  device, dt, [P][B][Lc][H][D]
 *   out[s][b][t][r*H/P + h'][:] = in[r][b][s*Lc+t][h'][:]
 * Bit-exact.  Errors as ra_ulysses_seq2head (H % P != 0 is RA_ERR_INVALID).
 */
RA_API ra_status ra_ulysses_head2seq(const void* in, void* out, int P, int B, int Lc,
                              int H, int D, ra_dtype dt, void* stream);

/*
 * ra_ulysses_seq2head_scatter / ra_ulysses_head2seq_scatter -- one rank's share of
 * the Ulysses all-to-all ([ULYSSES]: the exchange before attention and the one after
 * it) as a single kernel that stores each destination rank's block straight into that
 * rank's buffer: the pack, the all-to-all and the unpack in one pass.  Across GPUs the
 * dst pointers are the peers' buffers mapped into this process (symmetric memory);
 * on one GPU they may be local buffers.  After every rank r of the P has made its call
 * and a cross-rank barrier ordered after those calls has completed, rank r's buffer
 * holds exactly what ra_ulysses_seq2head / ra_ulysses_head2seq would give rank r.
 *   seq2head: in  device, dt, [B][Lc][H_in][D]: this rank's sequence shard s = rank.
 *             dst host array of P device pointers; dst[r] is rank r's [B][P*Lc][H_out/P][D]
 *             buffer, of which this call writes tokens rank*Lc .. rank*Lc + Lc - 1:
 *             dst[r][b][rank*Lc+t][h'][:] = in[b][t][floor((r*H_out/P + h')*H_in/H_out)][:]
 *   head2seq: in  device, dt, [B][P*Lc][H/P][D]: this rank's head group g = rank.
 *             dst[r] is rank r's [B][Lc][H][D] buffer, of which this call writes heads
 *             rank*H/P .. rank*H/P + H/P - 1:
 *             dst[r][b][t][rank*H/P + h'][:] = in[b][r*Lc+t][h'][:]
 * Plain 16-byte loads and stores (no TMA, no multicast); the kernel ends with a
 * system-scope fence.  Bit-exact.  The buffers are the caller's; the library frees and
 * synchronises nothing across ranks: the caller orders the calls against the readers
 * of the buffers (a barrier before, so that no rank is still reading its buffer, and one
 * after).  Asynchronous on stream.
 * Errors: as ra_ulysses_seq2head / ra_ulysses_head2seq with P ranks, and RA_ERR_INVALID
 *   for P outside [1, RA_MAX_P], rank outside [0, P), a null dst array, a null or
 *   misaligned dst[r], a dst[r] equal to in, or two equal dst pointers.
 */
RA_API ra_status ra_ulysses_seq2head_scatter(const void* in, void* const* dst, int P, int rank,
                                             int B, int Lc, int H_in, int H_out, int D,
                                             ra_dtype dt, void* stream);
RA_API ra_status ra_ulysses_head2seq_scatter(const void* in, void* const* dst, int P, int rank,
                                             int B, int Lc, int H, int D, ra_dtype dt,
                                             void* stream);

/*
 * ra_ulysses_replica_sum -- the gradient of seq->head's GQA copy ([ULYSSES]: KV heads are
 * copied so that every rank holds one): replica j of H_in = H_out * rep heads is a copy of
 * head j / rep, so the gradient of head g is the sum of the gradients of its rep replicas.
 *   in   device, fp32, [rows][H_in][D] (for example dK of the replicated heads, after
 *        head->seq: rows = B * Lc)
 *   out  device, fp32, [rows][H_out][D]
 *   out[r][g][:] = sum_{k < rep} in[r][g*rep + k][:], the replicas added in ascending k
 *   (the same bits on every call).  Caller-owned buffers; asynchronous on stream.
 * Errors: RA_ERR_INVALID for sizes < 1, H_in % H_out != 0, D % 4 != 0, null or
 *   misaligned (16-byte) pointers, in == out.
 */
RA_API ra_status ra_ulysses_replica_sum(const float* in, float* out, long long rows, int H_in,
                                        int H_out, int D, void* stream);

/*
 * ra_ulysses_seq2head_grouped / ra_ulysses_head2seq_grouped -- the two
 * transforms above with the head groups counted apart from the shards: G
 * groups of H_out/G heads, each receiving the tokens of all P shards.  G = P is
 * ra_ulysses_seq2head / ra_ulysses_head2seq.  G < P is the head split of the
 * ring x Ulysses hybrid (USP; [ACCEL-SP] names it beside Ulysses, and the ring
 * of [SP-QA] section 3 runs over the rest): with P = P_r * P_u virtual ranks,
 * the Ulysses all-to-all inside each group of P_u ranks leaves head group g with
 * the whole sequence, which ra_ring_attn_fwd then treats as P_r ring chunks.
 *   seq2head: in [P][B][Lc][H_in][D] -> out [G][B][P*Lc][H_out/G][D]
 *     out[g][b][s*Lc+t][h'][:] = in[s][b][t][floor((g*H_out/G + h')*H_in/H_out)][:]
 *   head2seq: in [G][B][P*Lc][H/G][D] -> out [P][B][Lc][H][D]
 *     out[s][b][t][g*H/G + h'][:] = in[g][b][s*Lc+t][h'][:]
 * Bit-exact.  Errors as the ungrouped forms, with G in place of P in the head
 * divisibility rules (H_out % G, H % G); RA_ERR_INVALID for G < 1.
 */
RA_API ra_status ra_ulysses_seq2head_grouped(const void* in, void* out, int P, int G, int B,
                                             int Lc, int H_in, int H_out, int D, ra_dtype dt,
                                             void* stream);
RA_API ra_status ra_ulysses_head2seq_grouped(const void* in, void* out, int P, int G, int B,
                                             int Lc, int H, int D, ra_dtype dt, void* stream);

/*
 * ra_sync_status -- synchronise `stream`, then read and clear this device's
 * kernel error word.  Returns RA_ERR_TIMEOUT if a kernel launched since the
 * last call gave up on a bounded wait, RA_ERR_CUDA if the synchronisation
 * itself failed, RA_OK otherwise.
 */
RA_API ra_status ra_sync_status(void* stream);

/* Thread-local description of the last non-OK status returned on this thread. */
RA_API const char* ra_last_error(void);

/*
 * ra_set_wait_limit_ns -- bound, in nanoseconds, on every internal spin-wait of
 * the tensor-core attention kernel (default 4e9).  Takes effect at the next
 * launch.  Returns the previous value.  ns == 0 restores the default.
 */
RA_API unsigned long long ra_set_wait_limit_ns(unsigned long long ns);

/*
 * ra_set_bwd_deterministic -- process-wide switch of every backward entry point
 * (ra_ring_attn_bwd and its _accumulate, _static, _zigzag and _packed forms).  With on != 0
 * the gradients are bitwise reproducible: dq comes from a kernel that keeps a query
 * tile stationary, visits the key tiles it sees in one fixed order and writes each dq
 * element once (adding it into dq in the _accumulate form), and the key-stationary
 * kernel computes dk and dv only.  It costs a second pass over the score tiles (1.2 to
 * 1.3 times the default backward's time, measured).  With on == 0 (the default) dq is
 * reduce-added from the key-stationary kernel, reproducible up to the rounding of
 * its fp32 sum.  Returns the previous setting (0 or 1).  Thread-safe; a call in
 * flight keeps the setting it started with.
 */
RA_API int ra_set_bwd_deterministic(int on);

/*
 * ra_debug_inject_stall -- test hook.  With on != 0 the next tensor-core
 * attention launch on this thread withholds one K tile load, so the consumer's
 * bounded wait expires, the kernel drains and exits, and ra_sync_status()
 * returns RA_ERR_TIMEOUT.  No fault and no unbounded wait is involved.  The
 * hook disarms itself after that launch.
 */
RA_API void ra_debug_inject_stall(int on);

/* Library version string. */
RA_API const char* ra_version(void);

#ifdef __cplusplus
}
#endif
#endif /* RA_B200_H */
