/*
 * sp.h -- C ABI of libsp, Ulysses sequence-parallel self-attention on one
 * B200 (sm_100a) with P virtual ranks.
 *
 * The method (fal.ai, "Generate video with WAN 2.2 across four GPUs",
 * section "Splitting one generation across four GPUs"): the token sequence
 * of one generation is split across P ranks; at each attention layer an
 * all-to-all exchanges token shards for head groups, so that every rank
 * attends over all tokens for H/P of the H heads, and the outputs go back to
 * the ranks that own the tokens.  The result is the single-GPU result
 * (LTX-2 "Multi-GPU Inference" README, Capabilities table).  On one GPU the exchange is a permutation in HBM
 * (sp_pack / sp_unpack) or disappears into the attention kernel's addressing
 * (sp_attention_seqsharded).  With one GPU per rank, sp_exchange_pack /
 * sp_exchange_unpack reorder a rank's shard around an all-to-all, and
 * sp_attention_ulysses_peer moves the Q and O exchanges into the attention
 * kernel over peer memory.
 *
 * Notation: B batch, N true token count, H heads, D head dim, P degree,
 * Hl = H/P, Nl = ceil(N/P), Np = P*Nl.  Elements are bf16 (16-bit words).
 *
 * Layouts (all dense, row-major, innermost last):
 *   sequence-sharded  xs : [P][B][Nl][H][D]   rank r holds tokens r*Nl .. r*Nl+Nl-1
 *   head-sharded      xh : [P][B][Np][Hl][D]  group j holds heads j*Hl .. j*Hl+Hl-1
 *   log-sum-exp      lse : [B][H][Np] fp32 (natural log), optional
 * Token slots t >= N are padding: they must be zero in xs for the pack to be
 * an exact copy of a zero-padded sequence; attention ignores them as keys and
 * writes zero output rows (lse = -inf) for them as queries.
 *
 * Ownership: the caller owns every buffer.  The library allocates no device
 * memory and keeps no pointer after a call returns.
 * Asynchrony: every call that takes a stream only enqueues work on it (NULL
 * means the legacy default stream) and does not synchronise, except
 * sp_device_status.
 * Errors: argument errors are returned before anything is enqueued and leave
 * the outputs untouched.  A failed launch returns SP_ERR_CUDA.  A kernel that
 * gives up on a bounded wait records SP_ERR_TIMEOUT in a device status word,
 * which sp_device_status reports.  Nothing throws across this ABI.
 * Requirements: device pointers 16-byte aligned; D in {64, 128};
 * H % P == 0; N >= 1; B >= 1; element counts below 2^31 per tensor row
 * index space.
 */
#ifndef SP_H_
#define SP_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SP_OK = 0,
  SP_ERR_NULL = 1,                /* a required pointer is NULL */
  SP_ERR_SHAPE = 2,               /* B, N, H, D or P out of range */
  SP_ERR_HEADS_NOT_DIVISIBLE = 3, /* H % P != 0 */
  SP_ERR_ALIGN = 4,               /* a device pointer is not 16-byte aligned */
  SP_ERR_UNSUPPORTED_D = 5,       /* D not in {64, 128} */
  SP_ERR_CUDA = 6,                /* a CUDA runtime/driver call failed */
  SP_ERR_TIMEOUT = 7              /* a kernel gave up on a bounded wait */
} sp_status;

/* One problem.  scale <= 0 selects 1/sqrt(D). */
typedef struct {
  int32_t B, N, H, D, P;
  float scale;
} sp_shape;

/* Np = ceil(N/P) * P, the padded token count of both layouts; -1 when
 * N < 1 or P < 1. */
int64_t sp_padded_tokens(int32_t N, int32_t P);

/* Validates a shape against the rules above.  The degree rule of the fal.ai
 * page, section "Tuning cost and GPU count" (P has to be a divisor of H),
 * gives SP_ERR_HEADS_NOT_DIVISIBLE. */
sp_status sp_check_shape(const sp_shape *shape);

/* Shard: the logical sequence of one generation divided across the P ranks
 * (page section "Splitting one generation across four GPUs"), rank r
 * holding tokens r*Nl .. r*Nl+Nl-1; token slots at or past N are zero:
 *   xs[r][b][n][h][c] = x[b][r*Nl + n][h][c]   (r*Nl + n < N), else +0.0
 * x: device [B][N][H][D] bf16, read only.  xs: device [P][B][Nl][H][D],
 * written in full.  Bit-exact copy.  Any P >= 1 (no heads are split). */
sp_status sp_shard(const void *x, void *xs, const sp_shape *shape, void *stream);

/* Unshard: the inverse of sp_shard, padding slots dropped:
 *   x[b][t][h][c] = xs[t / Nl][b][t % Nl][h][c]
 * xs: device [P][B][Nl][H][D] bf16, read only.  x: device [B][N][H][D],
 * written in full.  Bit-exact copy. */
sp_status sp_unshard(const void *xs, void *x, const sp_shape *shape, void *stream);

/* Pack: sequence-sharded -> head-sharded, the send reorder plus all-to-all
 * of the page section "Splitting one generation across four GPUs":
 *   xh[j][b][r*Nl + n][hh][c] = xs[r][b][n][j*Hl + hh][c]
 * xs: device, [P][B][Nl][H][D] bf16, read only.  xh: device,
 * [P][B][Np][Hl][D] bf16, written in full.  Bit-exact copy.  xs and xh must
 * not overlap. */
sp_status sp_pack(const void *xs, void *xh, const sp_shape *shape, void *stream);

/* Unpack: head-sharded -> sequence-sharded (the outputs go back to the ranks
 * that own the tokens, same section); the inverse of sp_pack:
 *   os[r][b][n][j*Hl + hh][c] = oh[j][b][r*Nl + n][hh][c]
 * oh: device, [P][B][Np][Hl][D] bf16, read only.  os: device,
 * [P][B][Nl][H][D] bf16, written in full.  Bit-exact copy. */
sp_status sp_unpack(const void *oh, void *os, const sp_shape *shape, void *stream);

/* Exchange pack on one rank, for the form in which every rank is its own
 * GPU: the send-buffer reorder in front of the all-to-all (same page
 * section).  Rank r's shard becomes P send chunks, chunk j holding r's
 * tokens for head group j:
 *   send[j][b][n][hh][c] = xs_r[b][n][j*Hl + hh][c]
 * After an all-to-all that delivers chunk j of every rank to rank j, in rank
 * order, rank j holds [P][B][Nl][Hl][D]: the sequence-sharded layout of its
 * Hl heads, which sp_attention_seqsharded with shape {B, N, Hl, D, P}
 * attends directly.
 * xs_r: device [B][Nl][H][D] bf16, read only.  send: device
 * [P][B][Nl][Hl][D] bf16, written in full.  shape: the global problem
 * (H % P == 0).  Bit-exact copy. */
sp_status sp_exchange_pack(const void *xs_r, void *send, const sp_shape *shape, void *stream);

/* Exchange unpack on one rank (outputs back to the token owners): the
 * P chunks returned by the head groups, chunk j = group j's output for this
 * rank's tokens, become the rank's shard:
 *   os_r[b][n][j*Hl + hh][c] = recv[j][b][n][hh][c]
 * recv: device [P][B][Nl][Hl][D] bf16, read only.  os_r: device
 * [B][Nl][H][D] bf16, written in full.  Bit-exact copy. */
sp_status sp_exchange_unpack(const void *recv, void *os_r, const sp_shape *shape, void *stream);

/* Attention per head group on head-sharded tensors: for every batch b,
 * group j, local head hh (global head h = j*Hl + hh) and query token i < N,
 *   oh[j][b][i][hh] = sum_{k<N} softmax_k(q_i . k_k * scale) v_k
 * non-causal, keys k >= N masked; every rank attends over all tokens for
 * its heads (same section).  Accumulation in fp32, probabilities rounded to
 * bf16 before the P*V product, output rounded to nearest-even bf16.  Rows
 * i in [N, Np) are written as zero.  The result for a given (b, h, i) does
 * not depend on P.
 * qh, kh, vh: device [P][B][Np][Hl][D] bf16, read only.  oh: device, same
 * shape, written.  lse: device fp32 [B][H][Np] or NULL. */
sp_status sp_attention(const void *qh, const void *kh, const void *vh, void *oh,
                       float *lse, const sp_shape *shape, void *stream);

/* Fused sequence-parallel attention: sp_unpack(sp_attention(sp_pack(q),
 * sp_pack(k), sp_pack(v))) in one kernel that reads Q/K/V tiles straight
 * from the sequence-sharded buffers and writes O into the sequence-sharded
 * layout; no intermediate buffers.  Bit-identical to the three-call path.
 * qs, ks, vs: device [P][B][Nl][H][D] bf16, read only.  os: device, same
 * shape, written.  lse: device fp32 [B][H][Np] or NULL.  With B > 1 and
 * P > 1 a token tile that crosses a shard boundary is gathered row by row
 * (slower than the TMA path used for every other tile and shape); padding
 * slots of qs/ks/vs must then be zero, as for sp_pack.  P describes only
 * how the tokens are sharded (no heads are split), so H % P == 0 is not
 * required here. */
sp_status sp_attention_seqsharded(const void *qs, const void *ks, const void *vs,
                                  void *os, float *lse, const sp_shape *shape,
                                  void *stream);

/* Tokens per scale block of the FP8 call's Q and K factors. */
#define SP_FP8_BLOCK 128

/* FP8 variant of sp_attention_seqsharded: Q, K and V in OCP E4M3, one byte
 * per element, each element scaled by a factor: Q and K element (b, t, h, c)
 * by q_scale / k_scale [b][h][t / SP_FP8_BLOCK], V element (b, t, h, c) by
 * v_scale[b][h][c].  The output O is bf16 as for the bf16 call.  QK^T and PV
 * run on the tensor cores' 8-bit path with fp32 accumulation; the
 * probabilities are rounded to E4M3 (relative rounding error at most 2^-4)
 * before the PV product, scaled by 2^6 relative to the running row maximum
 * so that the typical weights of long sequences keep E4M3's 3 mantissa bits.
 * The pages name FP8 and FP4 attention (FastVideo, "Pair two NVIDIA DGX
 * Sparks", the NVFP4 stacks) without defining it; this is the plainest
 * reading: the same attention on dequantized 8-bit inputs, with factors at
 * the granularity the two products allow (q.k sums over channels, so Q and K
 * factors may change from token block to token block; p.v sums over tokens,
 * so V factors may change from channel to channel).
 * qs, ks, vs: device [P][B][Nl][H][D] uint8 (E4M3), read only, 16-byte
 * aligned; D must be 128.  q_scale, k_scale: device fp32
 * [B][H][ceil(N / SP_FP8_BLOCK)]; v_scale: device fp32 [B][H][D]; all read
 * only, 4-byte aligned, finite and positive.  os: device [P][B][Nl][H][D]
 * bf16, written.  lse: device fp32 [B][H][Np] or NULL (natural log of the
 * row sum of exp(scaled logits)).  Results do not depend on P
 * (bit-identical).  Errors: SP_ERR_NULL for a NULL scale pointer, otherwise
 * as for sp_attention_seqsharded. */
sp_status sp_attention_fp8_seqsharded(const void *qs, const void *ks, const void *vs,
                                      const float *q_scale, const float *k_scale,
                                      const float *v_scale, void *os, float *lse,
                                      const sp_shape *shape, void *stream);

/* Where sp_qkv_projection writes q, k and v. */
typedef enum {
  SP_QKV_SEQ_SHARDED = 0,  /* [P][B][Nl][H][D]: the fused attention's input */
  SP_QKV_HEAD_SHARDED = 1, /* [P][B][Np][Hl][D]: sp_attention's input (the pack folded in) */
  SP_QKV_SEND_CHUNKS = 2   /* [P][B][Nl][Hl][D] of one rank: its exchange pack folded in */
} sp_qkv_layout;

/* The projection in front of attention: each token's hidden state to its q,
 * k and v, y[m][c] = sum_k x[m][k] * w[c][k] (+ bias[c]) with the 3*H*D output
 * features ordered q, k, v (head-major, D per head) and a feature's weights in
 * one row of w, as a linear layer stores them.  The pages never describe the
 * transformer block around the attention; this is its plainest reading (no
 * rotary embedding or normalisation).  The epilogue stores y straight into
 * the layout `layout` names, so no permutation pass runs between the
 * projection and attention.  fp32 accumulation, bf16 output (round to
 * nearest even).
 * x: device bf16 [P][B][Nl][hidden], the sequence-sharded hidden states
 *   (padding slots included), or for SP_QKV_SEND_CHUNKS one rank's
 *   [B][Nl][hidden]; 16-byte aligned; hidden a multiple of 8.
 * w: device bf16 [3*H*D][hidden]; bias: device bf16 [3*H*D] or NULL.
 * q, k, v: device bf16 outputs in `layout`, 16-byte aligned, written in full
 *   (padding slots hold the projection of x's padding rows).
 * shape: {B, N, H, D, P}; the head-split layouts need H % P == 0.
 * Errors: SP_ERR_NULL, SP_ERR_ALIGN, SP_ERR_SHAPE (layout, hidden, sizes),
 * SP_ERR_HEADS_NOT_DIVISIBLE, SP_ERR_UNSUPPORTED_D, SP_ERR_CUDA. */
sp_status sp_qkv_projection(const void *x, const void *w, const void *bias, void *q, void *k,
                            void *v, int32_t hidden, int32_t layout, const sp_shape *shape,
                            void *stream);

/* Where sp_out_projection reads the attention output O. */
typedef enum {
  SP_O_SEQ_SHARDED = 0,  /* [P][B][Nl][H][D]: the fused attention's output */
  SP_O_HEAD_SHARDED = 1, /* [P][B][Np][Hl][D]: sp_attention's output (the unpack folded in) */
  SP_O_RECV_CHUNKS = 2   /* [P][B][Nl][Hl][D] of one rank: the P chunks returned to it
                            (its exchange unpack folded in) */
} sp_o_layout;

/* The projection after attention: each token's attention output (all H
 * heads, H*D features, head-major) to its hidden state,
 *   y[m][c] = sum_k o[m][k] * w[c][k] (+ bias[c]),   k = h*D + d,
 * with a feature's weights in one row of w, as a linear layer stores them.
 * The pages place sequence parallelism inside the transformer block (LTX-2
 * "Multi-GPU Inference" README, section "Pages": the SP builder and its
 * attention manager swap in per block) but never describe the block; this is
 * the plainest reading of the step after attention (one linear layer).  The
 * layout work is folded into the operand loads: O is read in the layout
 * `layout` names, so neither sp_unpack nor sp_exchange_unpack runs between
 * attention and this projection.  fp32 accumulation, bf16 output (round to
 * nearest even).
 * o: device bf16 in `layout`, 16-byte aligned, read only.
 * w: device bf16 [hidden][H*D]; bias: device bf16 [hidden] or NULL.
 * y: device bf16 [P][B][Nl][hidden], the sequence-sharded hidden states
 *   (one rank's [B][Nl][hidden] for SP_O_RECV_CHUNKS), 16-byte aligned,
 *   written in full (padding slots hold the projection of O's padding rows,
 *   which attention writes as zero).
 * hidden: a multiple of 8.  shape: {B, N, H, D, P}; the head-split layouts
 *   need H % P == 0.
 * Errors: SP_ERR_NULL, SP_ERR_ALIGN, SP_ERR_SHAPE (layout, hidden, sizes),
 * SP_ERR_HEADS_NOT_DIVISIBLE, SP_ERR_UNSUPPORTED_D, SP_ERR_CUDA.  The result
 * does not depend on the layout (bit for bit). */
sp_status sp_out_projection(const void *o, const void *w, const void *bias, void *y,
                            int32_t hidden, int32_t layout, const sp_shape *shape, void *stream);

/* Tokens per cube of the block-sparse call's mask, and the most cubes
 * (ceil(N / SP_SPARSE_CUBE)) the call takes: 524,288 tokens. */
#define SP_SPARSE_CUBE 64
#define SP_SPARSE_MAX_CUBES 8192

/* Block-sparse variant of sp_attention_seqsharded: the sparse stage of video
 * sparse attention, which the FastVideo page ("Pair two NVIDIA DGX Sparks",
 * the FastH3 release stacks) runs with 64-token tiles and sparsity 0.8 but
 * whose block selection it does not define.  The selection is the caller's:
 * query token i attends key token t only when the mask selects t's cube for
 * i's cube (cubes of SP_SPARSE_CUBE consecutive tokens of the logical
 * sequence).  A query whose cube selects no key gets a zero output row and
 * lse = -inf.
 * mask: device uint32 [B][H][ncube][nwords], ncube = ceil(N / 64),
 *   nwords = ceil(ncube / 32); bit c of word w in query cube qc's row selects
 *   key cube 32*w + c; bits for cubes >= ncube are ignored.  Read only,
 *   4-byte aligned.
 * qs, ks, vs, os, lse as for sp_attention_seqsharded; D must be 128 and
 * ceil(N / 64) <= SP_SPARSE_MAX_CUBES (SP_ERR_UNSUPPORTED_D / SP_ERR_SHAPE).  Each 128-row
 * query tile (two query cubes) visits only the key cubes that one of its two
 * query cubes selects, two cubes per 128-key step: first the cubes that the
 * neighbouring tile of its CTA (the next or previous 128 rows) also visits,
 * then its own, each group in increasing order.  A row's result depends on
 * the mask rows of its CTA's four query cubes (through that order), never on
 * P or the layout.  With every cube selected the result equals
 * sp_attention_seqsharded's bit for bit. */
sp_status sp_attention_sparse_seqsharded(const void *qs, const void *ks, const void *vs,
                                         const uint32_t *mask, void *os, float *lse,
                                         const sp_shape *shape, void *stream);

/* ---------------------------------------------------------------------
 * Multi-GPU form with the Q and O exchanges fused into the attention kernel.
 *
 * "Splitting one generation across four GPUs" (fal.ai, "Generate video with
 * WAN 2.2 across four GPUs") moves Q, K and V from token shards to head
 * groups before attention and O back afterwards; the LTX-2 "Multi-GPU
 * Inference" README (Requirements) names an all2all kernel over CUDA-IPC
 * peer buffers for it.  In this form each Q tile crosses NVLink once, read by
 * TMA straight from the rank that holds it, and each O row once, stored by
 * the epilogue straight into the rank that owns it; only K and V, which every
 * query tile of a head re-reads, are exchanged into local memory first
 * (sp_exchange_pack + an all-to-all).
 */

/* Most ranks the peer step addresses. */
#define SP_MAX_PEERS 8

/* One rank's attention step: rank `rank` (= j) attends head group j (heads
 * j*Hl .. j*Hl+Hl-1, Hl = H/P) over the full sequence.
 * q_shards: HOST array of P device addresses valid in this process (this
 *   rank's own buffer and the peers' buffers mapped with sp_ipc_open);
 *   q_shards[r] is rank r's Q shard [B][Nl][H][D] bf16, read only, 16-byte
 *   aligned.  Token t of the sequence is row t % Nl of rank t / Nl.
 * k_group, v_group: this rank's received K and V head group
 *   [P][B][Nl][Hl][D] bf16 (chunk r from rank r), local, read only.
 * o_shards: HOST array of P device addresses; o_shards[r] is rank r's output
 *   shard [B][Nl][H][D] bf16; the kernel writes the columns of heads
 *   j*Hl .. j*Hl+Hl-1 of every row (padding rows as +0.0) and nothing else.
 * lse: device fp32 [B][Hl][Np] of this head group, or NULL.
 * shape: the whole problem {B, N, H, D, P}; D must be 128, P <= SP_MAX_PEERS,
 *   H % P == 0, 0 <= rank < P (else SP_ERR_UNSUPPORTED_D / SP_ERR_SHAPE /
 *   SP_ERR_HEADS_NOT_DIVISIBLE).
 * Ordering is the caller's: every rank's Q must be complete before the
 * launch, and rank r may read its O only after every rank's step has
 * finished (an all-to-all that follows the Q writes, and a collective after
 * the step, order both).  The kernel ends with a system-scope fence.
 * Results equal sp_attention_seqsharded's bit for bit. */
sp_status sp_attention_ulysses_peer(const void *const *q_shards, const void *k_group,
                                    const void *v_group, void *const *o_shards, float *lse,
                                    int32_t rank, const sp_shape *shape, void *stream);

/* ---------------------------------------------------------------------
 * The same step with the K/V exchange overlapped with attention.
 *
 * In sp_attention_ulysses_peer, K and V reach the head groups through an
 * all-to-all before the attention kernel starts.  Here each rank stores its
 * K/V chunks straight into the head groups' buffers over peer memory
 * (sp_exchange_push: the send-buffer reorder fused with the transfer, no
 * send buffer and no all-to-all) and counts each finished piece in the
 * receiving rank's arrival counters; the attention kernel
 * (sp_attention_ulysses_overlap) walks key tiles in their fixed order and,
 * before loading the tiles of source rank r's chunk (and the Q tiles of rank
 * r's shard), waits with a bounded wait until r's counter shows that the
 * chunk has arrived.  No collective gates the attention launch: it waits
 * only for the chunks its tiles read, so peers' pushes still in flight (or
 * late) overlap attention on the chunks that have arrived.  The order of the
 * arithmetic is unchanged, so results equal sp_attention_seqsharded's bit
 * for bit.  A rank's push and attention run in one stream, push first: an
 * attention kernel must never wait for a push on its own GPU that could run
 * concurrently with it.
 * Protocol: every rank owns a counter array uint64 [P] (zeroed once, before
 * any rank's first push) and a received-group buffer for K and for V.  Step
 * e = 1, 2, ... of every rank: write Q into its Q shard, then
 * sp_exchange_push(..., epoch = e), then sp_attention_ulysses_overlap(...,
 * epoch = e), then a collective that follows every rank's attention kernel
 * (as for sp_attention_ulysses_peer) before the next step overwrites any
 * buffer a peer reads.
 */

/* Rank `rank` stores its K and V chunks for every head group j into rank
 * j's received groups at chunk slot `rank`:
 *   k_groups[j][rank][b][n][hh][c] = k_r[b][n][j*Hl + hh][c]   (v alike)
 * and adds its finished pieces to counts[j][rank] with release semantics at
 * system scope (after step e that counter holds e times the pieces of one
 * step).
 * k_r, v_r: this rank's shards [B][Nl][H][D] bf16, local, read only.
 * k_groups, v_groups: HOST arrays of P device addresses valid in this
 *   process (this rank's own buffers and the peers' mapped with sp_ipc_open);
 *   each [P][B][Nl][Hl][D] bf16, 16-byte aligned; only chunk slot `rank` is
 *   written.
 * counts: HOST array of P device addresses of each rank's uint64 [P]
 *   arrival counters, 8-byte aligned.
 * epoch: this step's number, >= 1.  shape: the whole problem; H % P == 0,
 *   P <= SP_MAX_PEERS, 0 <= rank < P.
 * Errors: SP_ERR_NULL, SP_ERR_ALIGN, SP_ERR_SHAPE (also epoch 0),
 * SP_ERR_HEADS_NOT_DIVISIBLE, SP_ERR_UNSUPPORTED_D, SP_ERR_CUDA. */
sp_status sp_exchange_push(const void *k_r, const void *v_r, void *const *k_groups,
                           void *const *v_groups, uint64_t *const *counts, uint64_t epoch,
                           int32_t rank, const sp_shape *shape, void *stream);

/* sp_attention_ulysses_peer on this rank's received groups while they
 * arrive: before loading key tiles or Q tiles of source rank r, the kernel
 * waits until counts[r] (this rank's own counter array, local, 8-byte
 * aligned) shows step `epoch`'s pieces of r's chunk, at most wait_ns
 * nanoseconds per wait (0: 2 s).  A wait that runs out stops the kernel:
 * its in-flight copies and MMAs are drained, nothing is left running, and
 * SP_ERR_TIMEOUT is recorded in the device status word (sp_device_status).
 * Other arguments and results as for sp_attention_ulysses_peer. */
sp_status sp_attention_ulysses_overlap(const void *const *q_shards, const void *k_group,
                                       const void *v_group, void *const *o_shards, float *lse,
                                       const uint64_t *counts, uint64_t epoch, uint64_t wait_ns,
                                       int32_t rank, const sp_shape *shape, void *stream);

/* Bytes of a CUDA IPC memory handle. */
#define SP_IPC_HANDLE_BYTES 64

/* Exports the device allocation that contains dev_ptr to other processes on
 * this node: writes its SP_IPC_HANDLE_BYTES-byte handle to handle_out (host)
 * and the offset of dev_ptr from the allocation's base to *offset_out. */
sp_status sp_ipc_export(const void *dev_ptr, void *handle_out, int64_t *offset_out);

/* Maps an allocation exported by another process (peer access enabled on
 * first use); *base_out receives its base address in this process.  Add the
 * exporter's offset to reach its buffer.  Unmap with sp_ipc_close. */
sp_status sp_ipc_open(const void *handle, void **base_out);

/* Unmaps an allocation mapped by sp_ipc_open. */
sp_status sp_ipc_close(void *base);

/* Head-slice copy, for pipelines that move a problem between host and device
 * one group of heads at a time (heads are independent, so a group of Hg
 * heads with P | Hg is a problem of its own): for every row r < rows and
 * head h < nh,
 *   dst[r][dst_h0 + h][0 .. D-1] = src[r][src_h0 + h][0 .. D-1]
 * where a dst row holds dst_heads and a src row src_heads heads of D bf16
 * elements (rows = P*B*Nl for the sequence-sharded layout).  dst and src are
 * each device memory or page-locked host memory; the direction follows from
 * the pointers (unified addressing).  Enqueues one strided copy on `stream`
 * and no kernel; rows == 0 enqueues nothing.  Bit-exact.  Errors: SP_ERR_NULL;
 * SP_ERR_SHAPE when rows < 0, nh < 1, D < 1, a slice reaches past its row
 * (h0 < 0 or h0 + nh > heads) or a row is 2^31 bytes or more; SP_ERR_CUDA
 * when the copy cannot be enqueued. */
sp_status sp_copy_heads(void *dst, int32_t dst_heads, int32_t dst_h0, const void *src,
                        int32_t src_heads, int32_t src_h0, int64_t rows, int32_t nh,
                        int32_t D, void *stream);

/* Takes the device status word of the current device and clears it in one
 * atomic exchange enqueued on `stream`, then synchronises `stream` and
 * returns what it took: SP_ERR_TIMEOUT if a kernel gave up on a bounded wait
 * since the last call, SP_ERR_CUDA if the stream reports an error, else
 * SP_OK.  The word is shared by every stream of the device: a timeout that a
 * kernel on another stream records after the exchange is reported by the
 * next call, never lost.  Synchronise every stream that launched sp kernels
 * first to have all of them covered by this call. */
sp_status sp_device_status(void *stream);

/* Self-test of the bounded waits and of the abort path: enqueues one small
 * kernel that starts a bulk copy into shared memory and one tensor-core MMA,
 * then waits on a shared-memory barrier nothing will complete, with a limit
 * of limit_ns nanoseconds (clamped to 1 s).  The wait runs out; the kernel
 * waits for the copy and the MMA it issued, releases its tensor memory,
 * records SP_ERR_TIMEOUT in the device status word and returns; the next
 * sp_device_status call reports it (SP_ERR_CUDA if the drain did not
 * finish).  No GPU fault is involved. */
sp_status sp_selftest_wait_timeout(uint64_t limit_ns, void *stream);

/* Number of kernels this library has enqueued since it was loaded. */
uint64_t sp_launch_count(void);

/* Static description of a status code; never NULL. */
const char *sp_status_str(sp_status status);

#ifdef __cplusplus
}
#endif

#endif /* SP_H_ */
