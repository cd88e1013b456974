/*
 * lad.h — C ABI of the hybrid-attention decode library (sm_100a / B200).
 *
 * The library computes the attention hot path of a 7:1 KDA : gated-MLA hybrid model of the
 * Ling-3.1-flash kind, as described on two pages:
 *   [P1] "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B model need at 1M
 *        tokens?" (dev.to)
 *   [P2] "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers"
 *        (ai.thesatyajit.com)
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller. No call allocates device
 *     memory; where scratch space is needed the caller passes a workspace whose size a
 *     *_workspace_size() query returns. The library's only device-resident state is fixed-size
 *     and compiled in: one error word per kernel module (set by bounded waits and device-side
 *     input checks, read and cleared by lad_device_error()) and the scratch array of
 *     mla_latent_decode_noalloc (below).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every
 *     call only enqueues work and returns; results are ready when that stream reaches that
 *     point. One call forks part of its work onto a stream of its own and joins it back by
 *     events (kda_prefill_chunked with a workspace: one stream and three events per device,
 *     created at the first such call and kept for the process).
 *   - Tensors are dense, row-major, in the index order written next to each argument.
 *     bf16 tensors hold IEEE bfloat16 bit patterns (lad_bf16); fp32 tensors hold float.
 *   - Return value: LAD_OK (0) or a negative status. On error nothing was launched, except
 *     LAD_ECUDA from a launch, where the CUDA error is recorded in the message.
 *     lad_last_error() returns a description of the calling thread's last error.
 *   - Kernels that wait on on-chip barriers bound every wait; a wait that runs out sets a
 *     device-side error word (read with lad_device_error()) and the kernel returns early
 *     instead of hanging. Outputs of such a launch are undefined.
 */
#ifndef LAD_H
#define LAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t lad_bf16; /* IEEE bfloat16 bit pattern */

/* status codes */
#define LAD_OK 0
#define LAD_EINVAL (-1)        /* null pointer, negative or inconsistent size */
#define LAD_EUNSUPPORTED (-2)  /* a size or alignment the library does not implement */
#define LAD_ECUDA (-3)         /* a CUDA runtime error (launch, attribute, device query) */
#define LAD_EWORKSPACE (-4)    /* workspace missing or smaller than the query returned */

/* flags */
#define LAD_FLAG_SILU (1u << 0)      /* kda_conv_update: apply SiLU to the conv output */
#define LAD_FLAG_L2NORM_QK (1u << 1) /* KDA calls: L2-normalise q and k per head in fp32 first */
#define LAD_FLAG_OUT_FP32 (1u << 2)  /* KDA and MLA calls: write o as fp32 instead of bf16 */
#define LAD_FLAG_KEEP_STATE (1u << 3) /* kda_decode_multi: read S but do not write it back */
#define LAD_FLAG_ROPE_INTERLEAVED (1u << 4) /* RoPE calls: pair dims (2i, 2i+1) instead of (i, i+32) */
/* kda_decode_step, kda_conv_decode_step(_gated): launch as a programmatic dependent of the kernel
 * before this call on the stream. The call's CTAs may start, and read the state S, while that
 * kernel still runs; they read everything else (q, k, v or x, the conv tails, alpha, beta, the
 * gate) and write anything only once it has finished and its writes are visible. The caller
 * guarantees that the kernel launched just before this call on the stream does not write S (it
 * may be another layer's call; it must not be this state's previous step). Every kernel before
 * that one has finished before this call starts. */
#define LAD_FLAG_OVERLAP_PREV (1u << 5)

/* Description of the calling thread's most recent error ("" if none). */
const char *lad_last_error(void);

/* Library ABI version (major * 100 + minor). */
int lad_version(void);

/*
 * Reads and clears the device-side error word that bounded waits set (see above), after
 * synchronising `stream`. *code receives 0 when no kernel gave up a wait, else a nonzero tag
 * naming the kernel and the wait (0x101-0x104 and 0x107 latent decode, 0x201 chunked prefill,
 * 0x501 the KDA decode step's copy of a second head's state, taken at small batch),
 * 0x106 when an FP8-cache decode met a query value beyond the f16 range, 0x105 when
 * a paged decode met a block-table entry outside the pool, or 0x301 when mla_cache_append had a
 * position with no row to write. Returns LAD_OK or LAD_ECUDA.
 */
int lad_device_error(void *stream, int *code);

/*
 * lad_check_bounded_wait — a check of the failure handling above that faults nothing: it launches
 * one CTA of two warps on `stream` whose barrier waits can never complete (nothing arrives on
 * them). Warp 0's wait runs out after the bounded-wait limit (about 1 s), records tag 0x401 and
 * raises the CTA's abort flag; warp 1, whose wait starts half a limit later, then returns at once
 * instead of reaching its own limit; the kernel returns and the context stays usable.
 * Synchronises `stream`.
 *   tag      receives the recorded device error tag (0x401 expected)
 *   results  int[4]: warp 0's wait result (0 = gave up), warp 1's wait result (0), milliseconds
 *            warp 1 waited (about half the limit), the abort flag (1)
 * Returns LAD_OK, LAD_EINVAL (null output) or LAD_ECUDA.
 */
int lad_check_bounded_wait(int *tag, int *results, void *stream);

/*
 * kda_conv_update — one decode step of the short causal depthwise convolution in front of
 * the KDA recurrence. [P2] "How KDA and MLA split the work": q, k and v come through a short
 * causal convolution of width 4; [P2] "Does 292 GiB fit on four Hopper GPUs?": the layer keeps
 * "convolution tails" (K-1 past inputs per channel).
 *
 * For every sequence b and channel c (the Cch channels are q|k|v, 3 x 8192 at the pages'
 * shape):
 *   y[b][c] = sum_{i<K-1} w[c][i] * tail[b][i][c] + w[c][K-1] * x[b][c]  (+ bias[c])
 *   y       = y * sigmoid(y)                       if flags & LAD_FLAG_SILU
 * then the tail drops its oldest row and appends x: tail[b][i] <- tail[b][i+1], tail[b][K-2] <- x[b].
 * Arithmetic is fp32; y is rounded once to bf16 (round to nearest even).
 *
 *   x         bf16 [B][Cch]       new token (read)
 *   conv_tail bf16 [B][K-1][Cch]  row 0 oldest (read and updated in place)
 *   w         bf16 [Cch][K]       taps; w[c][K-1] multiplies the newest input
 *   bias      bf16 [Cch] or NULL
 *   y         bf16 [B][Cch]       output; must not alias x or conv_tail
 * Supported: K == 4, Cch % 8 == 0, all pointers 16-byte aligned. B == 0 is a no-op.
 */
int kda_conv_update(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *w, const lad_bf16 *bias,
                    lad_bf16 *y, int B, int Cch, int K, unsigned flags, void *stream);

/*
 * kda_decode_step — one token of Kimi Delta Attention (gated delta rule) for B sequences and
 * H heads. [P2] "How KDA and MLA split the work": each head keeps a 128x128 state, decays it
 * channel by channel (alpha, per key channel) and writes the new key-value association with a
 * per-head strength beta; [P1] "Why would a model keep only 9 full-attention layers?": KDA
 * extends Gated DeltaNet with finer-grained gating. The page's display equation is lost; the
 * update implemented (decay first, then the delta correction from the decayed state, readout
 * after the write) is:
 *   S'  = Diag(alpha) S
 *   u   = beta * (v - S'^T k)
 *   S   = S' + k u^T
 *   o   = scale * S^T q
 * with q, k L2-normalised first (x / sqrt(sum x^2 + 1e-6), fp32) if flags & LAD_FLAG_L2NORM_QK.
 * All state arithmetic is fp32.
 *
 *   q, k      bf16, row (b, h) at q + b*qkv_batch_stride + h*dk     (read)
 *   v         bf16, row (b, h) at v + b*qkv_batch_stride + h*dv     (read)
 *   qkv_batch_stride  elements between sequences in q, k and v; 0 means dense [B][H][d].
 *             (Pass 3*H*d with q, k, v pointing into kda_conv_update's y to consume it directly.)
 *   alpha     fp32 [B][H][dk]     decay per key channel, in (0, 1]
 *   beta      fp32 [B][H]         write strength
 *   S         fp32 [B][H][dk][dv] state, rows = key channels (read and updated in place)
 *   o         [B][H][dv], bf16, or fp32 if flags & LAD_FLAG_OUT_FP32
 * flags: LAD_FLAG_L2NORM_QK, LAD_FLAG_OUT_FP32, LAD_FLAG_OVERLAP_PREV.
 * Supported: dk == dv == 128; S 16-byte aligned. B == 0 or H == 0 is a no-op.
 */
int kda_decode_step(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, long long qkv_batch_stride,
                    const float *alpha, const float *beta, float *S, void *o, int B, int H, int dk, int dv,
                    float scale, unsigned flags, void *stream);

/*
 * kda_conv_decode_step_gated — kda_conv_decode_step with the head's output gate applied to o in
 * the same kernel. [P2] "How KDA and MLA split the work": each KDA layer also projects an output
 * gate (a full-rank 4096 -> 8192 projection, one value per output channel). The page does not give
 * the gate's form; the reading is the gated RMSNorm of the published KDA, per head over its dv
 * outputs:
 *   o <- o / sqrt(mean(o^2) + eps) * norm_w * sigmoid(gate)
 *   gate    bf16 [B][H][dv], 8-byte aligned       gate logits for this token (read)
 *   norm_w  fp32 [dv] or NULL (all ones), 16-byte aligned   per-channel weight, shared by heads
 *   eps     finite, >= 0
 * The other arguments, flags and limits are kda_conv_decode_step's; `scale` scales o before the
 * norm (so it only matters through eps).
 */
int kda_conv_decode_step_gated(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w,
                               const lad_bf16 *conv_bias, const float *alpha, const float *beta, float *S,
                               const lad_bf16 *gate, const float *norm_w, float eps, void *o, int B, int H, int dk,
                               int dv, int K, float scale, unsigned flags, void *stream);

/*
 * kda_decode_multi — kda_decode_step for T consecutive tokens per sequence in one pass over the
 * state (read once, written once): the verification step of multi-token prediction, one token
 * plus the drafts ([P1] "What does that mean for serving?": the serving recipe runs MTP with 3
 * speculative tokens; [P2] "What is in the files": one MTP layer serves as the draft head;
 * [P2] "The serving numbers are not one experiment": acceptance length 2.13-2.61). For
 * t = 0 .. n_b - 1 the recurrence of
 * kda_decode_step runs token by token (decay, delta write, readout after the write), so the
 * result equals n_b calls of kda_decode_step, up to fp32 rounding order.
 *
 *   q, k, v   bf16 [B][T][H][dk]   (read)
 *   alpha     fp32 [B][T][H][dk]; beta fp32 [B][T][H]
 *   S         fp32 [B][H][dk][dv]  read; written with the state after the n_b tokens unless
 *             flags & LAD_FLAG_KEEP_STATE
 *   o         [B][T][H][dv] bf16 (fp32 with LAD_FLAG_OUT_FP32), or NULL for no outputs; only
 *             positions t < n_b are written
 *   n_tokens  int32 [B] device, or NULL for n_b = T: sequence b applies its first
 *             n_b = clamp(n_tokens[b], 0, T) tokens
 * A verify-then-commit cycle is one call with LAD_FLAG_KEEP_STATE (outputs for all drafts), then
 * one call with n_tokens = the accepted counts and o = NULL (state committed).
 * flags: LAD_FLAG_L2NORM_QK, LAD_FLAG_OUT_FP32, LAD_FLAG_KEEP_STATE.
 * Supported: dk == dv == 128, 0 <= T <= 8; S, q, k, v and alpha 16-byte aligned. B, H or T == 0
 * is a no-op.
 */
int kda_decode_multi(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, const float *alpha, const float *beta,
                     float *S, void *o, const int *n_tokens, int B, int T, int H, int dk, int dv, float scale,
                     unsigned flags, void *stream);

/*
 * kda_conv_decode_step — kda_conv_update and kda_decode_step of one KDA layer in one launch: the
 * short convolution of each head's q, k and v channels runs in the CTA that updates that head's
 * state ([P2] "How KDA and MLA split the work": q, k, v come through the width-4 short causal
 * convolution, then the gated delta rule). The conv output stays in fp32 (it is not rounded to
 * bf16 on the way, unlike the two-call path) and never touches HBM.
 *
 *   x          bf16 [B][3*H*dk]       raw token, channels q | k | v (read)
 *   conv_tail  bf16 [B][K-1][3*H*dk]  tails, oldest row first (read and updated in place)
 *   conv_w     bf16 [3*H*dk][K]       taps (8-byte aligned); conv_bias bf16 [3*H*dk] or NULL
 *   alpha, beta, S, o                 as in kda_decode_step
 * flags: LAD_FLAG_SILU (conv output through SiLU), LAD_FLAG_L2NORM_QK, LAD_FLAG_OUT_FP32,
 * LAD_FLAG_OVERLAP_PREV.
 * Supported: dk == dv == 128, K == 4. B == 0 or H == 0 is a no-op.
 */
int kda_conv_decode_step(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w, const lad_bf16 *conv_bias,
                         const float *alpha, const float *beta, float *S, void *o, int B, int H, int dk, int dv, int K,
                         float scale, unsigned flags, void *stream);

/*
 * kda_prefill_chunked — the same recurrence as kda_decode_step over T tokens per sequence,
 * computed chunk by chunk (chunk length `chunk`, a shorter last chunk allowed) in the WY / UT
 * form: inside a chunk with cumulative decays g_r = prod_{s<=r} alpha_s,
 *   A = strict_lower(diag(beta) (K*g) (K/g)^T),  Tm = (I + A)^-1,
 *   U = Tm diag(beta) (V - (K*g) S0),
 *   O = scale ((Q*g) S0 + lower((Q*g)(K/g)^T) U),
 *   S = Diag(g_last) S0 + (K * g_last/g)^T U.
 * The pages do not print this form; it is the recurrence above unrolled within a chunk.
 *
 *   q, k, alpha  [B][T][H][dk] (q, k bf16; alpha fp32)
 *   v            bf16 [B][T][H][dv]
 *   beta         fp32 [B][T][H]
 *   S            fp32 [B][H][dk][dv]  initial state in, final state out
 *   o            [B][T][H][dv] bf16, or fp32 if flags & LAD_FLAG_OUT_FP32
 *   workspace    NULL, or device scratch of ws_bytes >= kda_prefill_workspace_size(...),
 *                256-byte aligned (else LAD_EWORKSPACE), owned by the caller and not read or
 *                written by anything else until the call's work on `stream` is done. With it
 *                the call runs two kernels per segment of up to 128 chunks: every chunk's
 *                state-independent operands in parallel, written to the workspace as one
 *                74,240-byte record per (sequence, head, chunk); then the state chain alone.
 *                The chains run on a stream the library keeps per device (highest priority),
 *                ordered by events: the chain of segment s overlaps the operands of segment
 *                s + 1, and `stream` waits for the last chain before any later work on it. The
 *                call can be captured in a CUDA graph: make the first call on a device outside
 *                a capture (it creates that stream and its events), and while a captured call's
 *                capture is open, other threads' calls on the same device must wait for its end
 *                (the side stream belongs to the capture until then). Without a workspace, one
 *                kernel does both per chunk on `stream`. Same results within rounding.
 * Supported: dk == dv == 128, chunk == 64; flags LAD_FLAG_L2NORM_QK, LAD_FLAG_OUT_FP32.
 * alpha must keep prod(alpha) over one chunk above ~1e-30 per channel (fp32 range of 1/g); the
 * workspace path also needs every K g_last / g and K / g of a chunk inside the fp16 range.
 */
int kda_prefill_chunked(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, const float *alpha,
                        const float *beta, float *S, void *o, int B, int T, int H, int dk, int dv, int chunk,
                        float scale, unsigned flags, void *workspace, size_t ws_bytes, void *stream);
/* Workspace bytes of kda_prefill_chunked's two-kernel path: a 256-byte header (item counters,
 * one per segment, rounded up to 256 bytes) plus B * H * min(ceil(T / 64), 128) records of
 * 74,240 bytes, twice over when T spans more than one segment of 128 chunks (about 1.22 GB for
 * one sequence of 64 heads and more than 8,192 tokens); 0 for unsupported shapes. */
size_t kda_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk);

/*
 * mla_latent_decode — gated Multi-head Latent Attention for one query token per sequence over
 * the compressed latent cache. [P2] "How KDA and MLA split the work": ordinary softmax
 * attention over a compressed cache whose rows hold a 512-dim latent plus a 64-dim RoPE key,
 * and a sigmoid gate per head scales the result; [P1] "How big is the cache per token,
 * exactly?": the cached row is kv_lora_rank + qk_rope_head_dim = 576 bf16 elements, the way
 * latent-attention kernels cache it; [P1] "...plain multi-head attention would be absurd":
 * the per-head key is 192 wide, hence the usual scale 1/sqrt(192).
 * The query arrives absorbed (W_UK folded in, RoPE applied), d_latent + d_rope wide. For each
 * sequence b with L = seq_lens[b] rows and each head h:
 *   s_t = scale * <q[b][h], c_t>            over all d_latent + d_rope dims
 *   o   = sum_t softmax(s)_t * c_t[0:d_latent]
 *   o  *= sigmoid(gate_logits[b][h])        if gate_logits != NULL
 *   lse = log sum_t exp(s_t)                (natural log, before the gate) if lse_out != NULL
 * L == 0 gives o = 0 and lse = -inf. Scores and softmax are fp32; q.c and p.c run on the
 * tensor cores with bf16 operands and fp32 accumulation. Rows at or past L are read up to the
 * next multiple of 32 (and below Lmax) but may hold anything, NaN included: they get exactly
 * zero weight.
 *
 *   q           bf16 [B][Hq][d_latent + d_rope]
 *   cache       bf16, row t of sequence b at cache + b*cache_seq_stride + t*(d_latent+d_rope)
 *   cache_seq_stride  elements between sequences (>= Lmax*(d_latent+d_rope), multiple of 8)
 *   seq_lens    int32 [B] device, each in [0, Lmax]
 *   gate_logits fp32 [B][Hq] or NULL
 *   o           [B][Hq][d_latent] bf16, or fp32 if flags & LAD_FLAG_OUT_FP32
 *   lse_out     fp32 [B][Hq] or NULL
 *   workspace   device scratch, ws_bytes >= mla_latent_decode_workspace_size(B, Hq, d_latent, 0)
 * Supported: Hq == 64, d_latent == 512, d_rope == 64; cache and q 16-byte aligned; scale > 0.
 */
int mla_latent_decode(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride, const int *seq_lens,
                      const float *gate_logits, void *o, float *lse_out, int B, int Hq, int d_latent, int d_rope,
                      int Lmax, float scale, unsigned flags, void *workspace, size_t ws_bytes, void *stream);

/* Workspace bytes mla_latent_decode needs; num_sms == 0 queries the current device. */
size_t mla_latent_decode_workspace_size(int B, int Hq, int d_latent, int num_sms);

/*
 * mla_latent_decode_paged — mla_latent_decode over a paged latent cache, the layout serving
 * engines keep it in ([P2] "How KDA and MLA split the work" and [P1] "How big is the cache per
 * token, exactly?" define the row and the attention; paging moves rows and changes no
 * arithmetic). Results equal mla_latent_decode's on the same rows.
 *
 *   kv_pages     bf16 [num_pages][page_size][d_latent + d_rope], a pool of pages
 *   block_table  int32 [B][block_table_stride] device: rows [j*page_size, (j+1)*page_size) of
 *                sequence b are page block_table[b*block_table_stride + j]; entries past
 *                ceil(seq_lens[b] / page_size) are not read
 *   seq_lens     int32 [B] device, each <= block_table_stride * page_size
 *   q, gate_logits, o, lse_out, scale, flags, workspace: as for mla_latent_decode (the same
 *                workspace size query)
 * Supported: page_size a positive multiple of 32 (a 32-row tile never spans two pages);
 * num_pages * page_size < 2^31; kv_pages 16-byte aligned. Rows of the last page past the length
 * may hold anything (NaN included): they get exactly zero weight. A needed block-table entry
 * outside [0, num_pages) (or past the stride) makes its rows read as zeros and sets device
 * error 0x105 (lad_device_error); the launch itself still returns LAD_OK.
 */
int mla_latent_decode_paged(const lad_bf16 *q, const lad_bf16 *kv_pages, int num_pages, int page_size,
                            const int *block_table, int block_table_stride, const int *seq_lens,
                            const float *gate_logits, void *o, float *lse_out, int B, int Hq, int d_latent,
                            int d_rope, float scale, unsigned flags, void *workspace, size_t ws_bytes,
                            void *stream);

/*
 * mla_latent_decode_paged_rope — mla_latent_decode_paged with RoPE applied to the query inside
 * the kernel. [P2] "Context: 1M in the claims, 262,144 in the config": position enters only the
 * MLA layers, through 64 of each head's 192 query-key dimensions, with rope_theta 6e6 and no
 * scaling. q's last d_rope = 64 values per head arrive not yet turned; the kernel turns them to
 * positions[b] (the query token's position, normally seq_lens[b] - 1) before the scores. The
 * pairing is not on the pages: dims (i, i + 32) by default, (2i, 2i + 1) with
 * LAD_FLAG_ROPE_INTERLEAVED; pair i turns by positions[b] * rope_theta^(-2i/64) (angle and sines in
 * fp64, the turned values rounded to bf16 once). The cache rows are expected turned already, as
 * mla_cache_append writes them.
 *   positions  int32 [B] device; rope_theta > 1
 *   the rest   as for mla_latent_decode_paged; flags: LAD_FLAG_OUT_FP32, LAD_FLAG_ROPE_INTERLEAVED
 */
int mla_latent_decode_paged_rope(const lad_bf16 *q, const int *positions, float rope_theta, const lad_bf16 *kv_pages,
                                 int num_pages, int page_size, const int *block_table, int block_table_stride,
                                 const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B,
                                 int Hq, int d_latent, int d_rope, float scale, unsigned flags, void *workspace,
                                 size_t ws_bytes, void *stream);

/*
 * mla_cache_append — writes one new latent-cache row per sequence: [P1] "How big is the cache per
 * token, exactly?" (a row is the 512-wide compressed latent followed by the 64-wide RoPE key, bf16),
 * with the RoPE key turned to the token's position here ([P2] "Context: 1M in the claims, 262,144
 * in the config"; pairing and angles as in mla_latent_decode_paged_rope, computed in fp64, each
 * turned value rounded to bf16 once; the latent is stored as given).
 *   c_kv       bf16 [B][d_latent], 16-byte aligned    the compressed latent (after its norm)
 *   k_pe       bf16 [B][d_rope]                        the RoPE key, not yet turned
 *   positions  int32 [B] device                        row index of the new token in its sequence
 *   cache      bf16, 16-byte aligned: with block_table == NULL the contiguous cache of
 *              mla_latent_decode (row t of sequence b at b*cache_seq_stride + t*576, t < Lmax);
 *              otherwise the page pool of mla_latent_decode_paged (num_pages pages of page_size
 *              rows; row t of sequence b in page block_table[b*block_table_stride + t/page_size])
 * A position with no row to write (negative, >= Lmax, past the block table or naming a page outside
 * the pool) writes nothing and sets device error 0x301 (lad_device_error).
 * flags: LAD_FLAG_ROPE_INTERLEAVED. Supported: d_latent == 512, d_rope == 64; rope_theta > 1.
 */
int mla_cache_append(const lad_bf16 *c_kv, const lad_bf16 *k_pe, const int *positions, lad_bf16 *cache,
                     long long cache_seq_stride, int Lmax, const int *block_table, int block_table_stride,
                     int num_pages, int page_size, int B, int d_latent, int d_rope, float rope_theta, unsigned flags,
                     void *stream);

/*
 * mla_latent_decode_multi — the MLA half of a multi-token step (speculative-decoding verify, [P1]
 * "What does that mean for serving?" / [P2] "What is in the files": an MTP layer drafts 3 tokens).
 * T query tokens per sequence: the last T of sequence b's seq_lens[b] cached rows are the tokens'
 * own rows (appended first), and token j (0-based) attends rows 0 .. seq_lens[b] - T + j, a
 * causal reading the pages leave open. T = 1 is mla_latent_decode.
 *   q           bf16 [B][T][Hq][576]
 *   gate_logits fp32 [B][T][Hq] or NULL;  o [B][T][Hq][d_latent];  lse_out fp32 [B][T][Hq] or NULL
 *   cache, cache_seq_stride, seq_lens, Lmax, scale, flags: as for mla_latent_decode
 *   workspace   ws_bytes >= mla_latent_decode_multi_workspace_size(B, T, Hq, d_latent, 0), 256-aligned
 * Each token is attended as a sequence of its own over the shared rows (the cache is read once per
 * token from HBM or L2). Tokens with no row to attend (seq_lens[b] - T + j < 0) give o = 0, lse = -inf.
 */
int mla_latent_decode_multi(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride,
                            const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B, int T,
                            int Hq, int d_latent, int d_rope, int Lmax, float scale, unsigned flags, void *workspace,
                            size_t ws_bytes, void *stream);
size_t mla_latent_decode_multi_workspace_size(int B, int T, int Hq, int d_latent, int num_sms);

/*
 * FP8 latent cache. [P1] "How big is the cache per token, exactly?": the bf16 cache takes 2 bytes
 * per element and an FP8 cache would halve it; [P2] "Does 292 GiB fit on four Hopper GPUs?": an
 * FP8 cache doubles the tokens that fit. The FP8 the pages use is E4M3 ([P2] "What is in the
 * files", with one fp32 scale per weight block); for the cache they give no scale, and the
 * reading here is one fp32 scale per cache: element = kv_scale * E4M3(code). E4M3: sign, 4
 * exponent bits (bias 7), 3 mantissa bits, largest finite 448, 0x7F / 0xFF NaN, no infinity.
 *
 * mla_latent_decode_fp8 — mla_latent_decode over an FP8 cache. The codes are widened to f16
 * exactly on chip and the query is converted bf16 -> f16 (exact for |q| <= 65504 outside the f16
 * subnormal range; a larger |q| sets device error 0x106), so the tensor cores run q.c and p.c on
 * f16 operands with fp32 accumulation (P in f16); kv_scale is applied to the fp32 scores and to
 * the normalised output. A bounded wait of the widening warps that gives up sets 0x107.
 *   cache             E4M3 codes, row t of sequence b at cache + b*cache_seq_stride + t*576 (bytes)
 *   cache_seq_stride  bytes between sequences (>= Lmax*576, multiple of 16)
 *   kv_scale          > 0, finite
 *   the rest          as for mla_latent_decode (same workspace size query); rows at or past
 *                     seq_lens[b] are never read; rows at or past Lmax read as zeros
 * Supported: as mla_latent_decode; cache and q 16-byte aligned.
 */
int mla_latent_decode_fp8(const lad_bf16 *q, const uint8_t *cache, long long cache_seq_stride, float kv_scale,
                          const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B, int Hq,
                          int d_latent, int d_rope, int Lmax, float scale, unsigned flags, void *workspace,
                          size_t ws_bytes, void *stream);

/*
 * mla_latent_decode_paged_fp8 — mla_latent_decode_paged over a pool of FP8 pages, with the
 * query's RoPE part turned in the kernel when positions != NULL (as mla_latent_decode_paged_rope;
 * rope_theta is then > 1 and LAD_FLAG_ROPE_INTERLEAVED selects the pairing) or arriving turned
 * when positions == NULL (rope_theta ignored).
 *   kv_pages   E4M3 codes [num_pages][page_size][576], 16-byte aligned
 *   kv_scale   > 0, finite
 *   the rest   as for mla_latent_decode_paged (block table, limits, device error 0x105)
 */
int mla_latent_decode_paged_fp8(const lad_bf16 *q, const int *positions, float rope_theta, const uint8_t *kv_pages,
                                float kv_scale, int num_pages, int page_size, const int *block_table,
                                int block_table_stride, const int *seq_lens, const float *gate_logits, void *o,
                                float *lse_out, int B, int Hq, int d_latent, int d_rope, float scale, unsigned flags,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * mla_cache_append_fp8 — mla_cache_append into an FP8 cache: each element x of the new row (the
 * latent as given, the RoPE key turned in fp64) is stored as the E4M3 code of x / kv_scale, the
 * quotient taken in fp32 (x rounded to fp32 first; one IEEE division) and rounded to nearest
 * even, saturating at +-448 (NaN stays NaN).
 *   cache       E4M3 codes, 16-byte aligned; contiguous (cache_seq_stride in bytes, multiple
 *               of 16) or a page pool, as for mla_cache_append
 *   kv_scale    > 0, finite
 *   the rest    as for mla_cache_append (device error 0x301 for a position with no row)
 */
int mla_cache_append_fp8(const lad_bf16 *c_kv, const lad_bf16 *k_pe, const int *positions, uint8_t *cache,
                         long long cache_seq_stride, int Lmax, const int *block_table, int block_table_stride,
                         int num_pages, int page_size, int B, int d_latent, int d_rope, float rope_theta,
                         float kv_scale, unsigned flags, void *stream);

/*
 * mla_latent_decode_noalloc — mla_latent_decode for callers that cannot allocate device memory
 * (a plugin inside a runtime that owns every device allocation, or a decode loop where
 * cudaMalloc's implicit synchronisation is not allowed). The pages have no counterpart: this is
 * a property of the library, not of the method. Results equal mla_latent_decode's.
 *
 * The caller still passes all inputs and outputs (same meaning, layouts and limits as
 * mla_latent_decode); only the scratch space differs: it is a fixed array compiled into the
 * library (about 25 MB, allocated on every device that loads the library and held until the
 * process exits), so this call itself allocates nothing.
 *   - B must not exceed mla_latent_decode_noalloc_max_batch() (32); larger B returns
 *     LAD_EUNSUPPORTED with a message. The device must have at most 160 SMs.
 *   - The first call on a device looks up the array's device address (with that device
 *     current) and keeps it for the life of the process; make that first call before any stream
 *     capture, and do not reset the device (cudaDeviceReset) while the library is in use: a new
 *     primary context would leave the kept address stale.
 *   - All calls share the one array: calls whose kernels may overlap on the GPU (different
 *     streams, or different host threads) race and give undefined results. Serialise them.
 *   - The array keeps the last call's contents; nothing in it needs to start at zero.
 */
int mla_latent_decode_noalloc(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride,
                              const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B, int Hq,
                              int d_latent, int d_rope, int Lmax, float scale, unsigned flags, void *stream);
size_t mla_latent_decode_noalloc_max_batch(void);

#ifdef __cplusplus
}
#endif

#endif /* LAD_H */
