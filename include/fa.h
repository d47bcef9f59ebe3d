/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa_b200.so).
 *
 * Operation.  Exact scaled-dot-product attention (forward, and its backward in fa_bwd):
 *     O = softmax(scale * Q K^T [+ causal mask]) V,   LSE_i = log sum_j exp(scale * q_i . k_j)
 * computed tile by tile with a running row max and row sum, so the N x N score matrix never
 * leaves the chip ("Flash Attention" (velog.io/@myungum), section 2 and its pseudocode: blocks of
 * Q, K, V are loaded into on-chip memory, the row max m and row sum l are carried across key
 * blocks, and only O, l, m are written back; "How Flash Attention reduces memory traffic"
 * (zimaspace), tiling and online softmax).  Work is split over batch, head and query tile
 * ("FlashAttention-2 GPU work partitioning", section 3).  The paged entry points (decode, chunked
 * prefill, draft-tree verification) read keys and values through a block table that maps each
 * sequence's logical KV blocks to physical blocks of a shared pool ("LLM study notes"
 * (devocean.sk.com), paged attention).  Key-range partials and their merge serve a sequence whose
 * keys are split across devices.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never allocates,
 *     frees or synchronises device memory (except fa_get_device_status, which synchronises the
 *     given stream).  Every launch is asynchronous on the caller's stream.
 *   - bf16 inputs (IEEE bfloat16 bit patterns), fp32 accumulation.
 *   - Arguments are checked on the host before anything is launched; on error nothing runs and a
 *     status code is returned.  No entry point aborts, traps or prints.
 *   - Device-side waits are bounded: a kernel that stops making progress records FA_ERR_TIMEOUT in
 *     a device status word and returns; fa_get_device_status reports and clears it.
 *   - Thread safety: calls on different streams may run concurrently; the status word is shared.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fa_stream_t; /* the same handle as cudaStream_t; NULL = legacy default */

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* a size, pointer or scale is out of range                         */
    FA_ERR_UNSUPPORTED = 2, /* head dimension other than 64 or 128, or a non-B200 device        */
    FA_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned                                  */
    FA_ERR_LAUNCH = 4,      /* the CUDA launch failed; fa_last_error_string() has the CUDA text  */
    FA_ERR_TIMEOUT = 5,     /* a kernel gave up waiting (reported by fa_get_device_status)       */
    FA_ERR_WORKSPACE = 6    /* a workspace is NULL or smaller than required (decode, backward)   */
} fa_status;

typedef enum {
    FA_OUT_BF16 = 0, /* written as bf16 (round to nearest even) */
    FA_OUT_F32 = 1   /* written as fp32                          */
} fa_out_dtype;

/*
 * fa_fwd -- prefill / full-sequence attention forward.
 *
 * Defined by the plain attention of "LLM study notes", self-attention steps (dot product of query
 * and key, divide by sqrt(d_k), softmax, weight the values), evaluated with the tiled online
 * softmax of "Flash Attention" (myungum), section 2.  Causal: query i sees keys 0..i
 * ("FlashAttention-2 GPU work partitioning", section 4).
 *
 *   q, k, v   bf16 [B, H, N, d], contiguous (row i of head (b,h) at ((b*H + h)*N + i)*d).
 *             May alias one another.  16-byte aligned.
 *   o         [B, H, N, d] contiguous, bf16 or fp32 per o_dtype.  16-byte aligned.  Must not
 *             overlap q, k, v or lse.
 *   lse       fp32 [B, H, N] (natural log of the row sum of exp(scaled scores)), or NULL.
 *   B, H, N   >= 1;  B*H*N*d must fit in int64;  B*H < 2^31;  B*H*ceil(N/256) < 2^31;  N < 2^31.
 *   d         64 or 128 (else FA_ERR_UNSUPPORTED).
 *   causal    0 or 1.
 *   scale     > 0 and finite; pass 0 (or any value <= 0) for 1/sqrt(d).  NaN/inf -> INVALID_ARG.
 *   stream    the stream to launch on.
 * Returns FA_OK once the kernel is queued.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, fa_out_dtype o_dtype,
                 float *lse, int B, int H, int N, int d, int causal, float scale,
                 fa_stream_t stream);

/*
 * fa_fwd_keyrange -- attention of queries over one contiguous range of the same sequence's keys:
 * the partial that one device computes when a long sequence's keys and values are split across
 * devices (sequence-length parallelism, "FlashAttention-2 GPU work partitioning", section 3).
 *
 * Query row i of q (i in [q_row0, Nq)) sits at position i; key row c of k, v sits at position
 * k_pos0 + c.  causal = 1: a query sees the keys at positions <= its own; otherwise all Nk keys.
 * O and LSE are those of the plain row definition over the keys each query sees (normalised
 * within the range); a row that sees none of them gets O = 0 and LSE = -inf.  Rows < q_row0 of o
 * and lse are not touched.  Partials of disjoint ranges combine with fa_merge_partials.
 *
 *   q            bf16 [B, H, Nq, d];  k, v: bf16 [B, H, Nk, d];  16-byte aligned.
 *   o            [B, H, Nq, d], bf16 or fp32 per o_dtype (fp32 for partials to be merged);
 *                lse: fp32 [B, H, Nq] or NULL (needed for merging).  Must not overlap the inputs.
 *   B, H, Nq, Nk >= 1;  B*H*ceil(Nq/256) < 2^31;  0 <= q_row0 < Nq;  k_pos0 >= 0;  d: 64 or 128;
 *   causal 0/1;  scale as for fa_fwd.
 * Returns FA_OK once the kernels are queued.
 */
fa_status fa_fwd_keyrange(const void *q, const void *k, const void *v, void *o, fa_out_dtype o_dtype,
                          float *lse, int B, int H, int Nq, int q_row0, int Nk, int k_pos0, int d,
                          int causal, float scale, fa_stream_t stream);

/*
 * fa_merge_partials -- combine G attention partials of the same query rows over disjoint key
 * ranges, with the rescaling rule of "Flash Attention" (myungum), section 2, steps 11-12, in
 * log-sum-exp form: M = max_g LSE_g, w_g = exp(LSE_g - M), O = sum_g w_g O_g / sum_g w_g,
 * LSE = M + ln sum_g w_g (a row whose partials are all -inf gets O = 0, LSE = -inf).
 *
 *   o_parts      fp32 [G, rows, d] contiguous, 16-byte aligned;  lse_parts: fp32 [G, rows].
 *   o            [rows, d], bf16 or fp32 per o_dtype;  lse: fp32 [rows] or NULL.  Must not overlap
 *                the partials.
 *   G, rows >= 1;  d: 64 or 128.
 * Returns FA_OK once the kernel is queued.
 */
fa_status fa_merge_partials(const float *o_parts, const float *lse_parts, int G, long long rows,
                            int d, void *o, fa_out_dtype o_dtype, float *lse, fa_stream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs: 4 * (d + 2) per query row, with
 * N rounded up to a multiple of 128.  Returns 0 on invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- attention backward: the gradients dQ, dK, dV of sum(dO * O) for O = fa_fwd(q, k, v).
 *
 * The pages give the backward in prose only: gradients are computed block by block from the
 * intermediate results the forward kept ("Paged vs Flash attention", training), and the attention
 * matrix is recomputed rather than stored ("LLM study notes", FlashAttention; "Flash Attention"
 * (myungum), section 1).  The forward keeps LSE; P is recomputed tile by tile as
 * exp(scale q.k - LSE), and with D_i = sum_c dO[i,c] O[i,c]:
 *     dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 *   q, k, v, dout     bf16 [B, H, N, d] contiguous, 16-byte aligned; dout is the incoming gradient.
 *   o, o_dtype        fa_fwd's output for the same q, k, v, causal and scale, [B, H, N, d] in bf16
 *                     or fp32.  D is formed from it, so bf16 O carries its own rounding (up to
 *                     2^-8 relative) into dS; fp32 O avoids that where rows are nearly one-hot.
 *   lse               fp32 [B, H, N], fa_fwd's log-sum-exp for the same call.
 *   dq, dk, dv        [B, H, N, d], bf16 or fp32 per g_dtype, 16-byte aligned; must not overlap the
 *                     inputs, one another or the workspace.
 *   B, H, N, d, causal, scale   as for fa_fwd.
 *   workspace         device scratch of at least fa_bwd_workspace_size(B, H, N, d) bytes, 16-byte
 *                     aligned, owned by the caller; no initialisation needed, garbage afterwards.
 *                     Two calls in flight at once need separate workspaces.
 * Three kernels are queued on the stream (row statistics, the blockwise gradients, the dQ
 * conversion).  dQ is summed in fp32 with atomic adds, so its last bits may differ between runs;
 * dK and dV are deterministic.  Returns FA_OK once the kernels are queued.
 */
fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o, fa_out_dtype o_dtype,
                 const void *dout, const float *lse, void *dq, void *dk, void *dv,
                 fa_out_dtype g_dtype, int B, int H, int N, int d, int causal, float scale,
                 void *workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_decode_workspace_size -- bytes of device workspace fa_decode_paged needs for these sizes.
 * The split of each sequence's context into chunks depends only on the arguments here, so the
 * same values must be passed to fa_decode_paged.  Returns 0 on invalid sizes.
 */
size_t fa_decode_workspace_size(int num_seqs, int H, int d, int max_blocks_per_seq);

/*
 * fa_decode_paged -- one decode step (query length 1) over a paged KV cache.
 *
 * The cache is a pool of fixed 16-token blocks; sequence s's logical block t lives in physical
 * block block_table[s * max_blocks_per_seq + t] ("LLM study notes", paged attention: the block
 * table makes logically contiguous KV memory out of physically scattered blocks).  The query of
 * sequence s attends to its seq_lens[s] cached tokens (it sits after them, so nothing is masked).
 * The context is split into chunks processed in parallel; the per-chunk running max, sum and
 * unnormalised output are merged with the same rescaling rule the tiled algorithm uses between
 * key blocks ("Flash Attention" (myungum), section 2, the m_new / l_new update).
 *
 *   q            bf16 [S, H, d] contiguous.
 *   k_pool,
 *   v_pool       bf16 [num_blocks, H, 16, d] contiguous (one 16 x d block per (block, head)).
 *   block_table  int32 [S, max_blocks_per_seq], device; entries t < ceil(seq_lens[s]/16) must be
 *                in [0, num_blocks); later entries are never read.
 *   seq_lens     int32 [S], device; each in [1, 16 * max_blocks_per_seq].  Values are not
 *                checked on the host (they live on the device); out-of-range lengths are clamped
 *                to that interval by the kernel.
 *   o            [S, H, d], bf16 or fp32 per o_dtype;  lse: fp32 [S, H] or NULL.
 *   S, H         >= 1;  d: 64 or 128;  scale as for fa_fwd.
 *   workspace    device scratch of at least fa_decode_workspace_size(S, H, d, max_blocks_per_seq)
 *                bytes, 16-byte aligned, owned by the caller; its contents need no initialisation
 *                and are garbage afterwards.  Two calls in flight at once need separate workspaces.
 * Returns FA_OK once the kernels are queued.
 */
fa_status fa_decode_paged(const void *q, const void *k_pool, const void *v_pool,
                          const int32_t *block_table, int max_blocks_per_seq,
                          const int32_t *seq_lens, int num_blocks, void *o, fa_out_dtype o_dtype,
                          float *lse, int S, int H, int d, float scale, void *workspace,
                          size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_prefill_paged -- chunked prefill over a paged KV cache: a chunk of Lq new queries per
 * sequence attends to that sequence's cached keys and values, read through the block table.
 *
 * Paging for the cache, exact tiled attention for the compute ("Paged vs Flash attention", their
 * combination; "LLM study notes", paged attention: the block table maps a sequence's logical
 * blocks to physical ones).  The chunk is the last Lq of the sequence's L = seq_lens[s] cached
 * tokens (its keys and values are already in the cache), so query t sits at position L - Lq + t:
 * with causal = 1 it sees keys 0 .. L - Lq + t (the mask aligned to the bottom-right of the
 * L x Lq score block); with causal = 0 it sees all L keys.  Lq = 1 is the decode step.
 *
 *   q            bf16 [S, H, Lq, d] contiguous.
 *   k_pool,
 *   v_pool       bf16 [num_blocks, H, 16, d] contiguous.
 *   block_table  int32 [S, max_blocks_per_seq], device; entries for pages < ceil(L/16) must be in
 *                [0, num_blocks); later entries are never read.  A bad entry is reported through
 *                fa_get_device_status (FA_ERR_INVALID_ARG) and its page reads as zeros.
 *   seq_lens     int32 [S], device; each in [Lq, 16 * max_blocks_per_seq] (lengths outside are
 *                clamped into it and reported the same way).
 *   o            [S, H, Lq, d], bf16 or fp32 per o_dtype;  lse: fp32 [S, H, Lq] or NULL.
 *   S, H, Lq     >= 1, Lq <= 16 * max_blocks_per_seq;  d: 64 or 128;  causal 0/1;
 *                (num_blocks + 1) * H <= INT_MAX (else FA_ERR_INVALID_ARG).
 *   scale        as for fa_fwd.
 * Returns FA_OK once the kernel is queued.  No workspace.
 */
fa_status fa_prefill_paged(const void *q, const void *k_pool, const void *v_pool,
                           const int32_t *block_table, int max_blocks_per_seq,
                           const int32_t *seq_lens, int num_blocks, void *o, fa_out_dtype o_dtype,
                           float *lse, int S, int H, int Lq, int d, int causal, float scale,
                           fa_stream_t stream);

/*
 * fa_tree_attention -- verification step of speculative decoding: every node of a draft-token
 * tree is scored against the context and its own path through the tree, in one pass.
 *
 * The draft model proposes candidate tokens as a tree and the target model checks all of its
 * nodes in a single forward pass with tree attention ("LLM study notes", speculative decoding).
 * The tree's T nodes are the last T of sequence s's L = seq_lens[s] cached tokens, in topological
 * order (their keys and values already written).  Node t sees the L - T context tokens and node u
 * exactly when bit u of tree_mask[s * T + t] is set: its ancestors and itself for a tree, though
 * any mask over the T nodes is accepted.  A node that sees no key at all gets O = 0 and LSE = -inf.
 *
 *   q            bf16 [S, H, T, d] contiguous (the nodes' queries).
 *   k_pool, v_pool, block_table, max_blocks_per_seq, seq_lens, num_blocks, o, o_dtype, lse, d,
 *   scale        as for fa_prefill_paged with Lq = T (each seq_lens[s] >= T).
 *   tree_mask    uint64 [S, T], device, 8-byte aligned; must not overlap o.
 *   T            1 .. 64.
 * Returns FA_OK once the kernel is queued.  No workspace.
 */
fa_status fa_tree_attention(const void *q, const void *k_pool, const void *v_pool,
                            const int32_t *block_table, int max_blocks_per_seq,
                            const int32_t *seq_lens, int num_blocks, const uint64_t *tree_mask,
                            void *o, fa_out_dtype o_dtype, float *lse, int S, int H, int T, int d,
                            float scale, fa_stream_t stream);

/*
 * fa_decode_paged_noalloc -- fa_decode_paged without a caller-supplied workspace and without any
 * allocation.  No counterpart in the paper: this is a deployment variant of the same decode step,
 * not part of the method.
 *
 * Who needs it: callers that cannot call cudaMalloc at decode time -- for instance a serving
 * engine that has handed almost all device memory to its own KV-cache pool and allocator (a
 * cudaMalloc would fail or fragment that pool), or a decode loop that cannot afford the
 * device-wide synchronisation and latency that cudaMalloc/cudaFree may cost.  Such callers still
 * own q, the pools, the table, the lengths, o and lse; only the split-context scratch moves.
 *
 * The scratch is a static device array of FA_NOALLOC_SCRATCH_BYTES inside this library: every
 * GPU that loads the library holds it until the process exits.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress, no allocation) and keeps it for the
 * life of the process; make that first call before any stream capture.  A device reset
 * (cudaDeviceReset, or the primary context destroyed and created again) makes the kept address
 * stale: do not call this entry point again in a process after resetting a device it has run on.
 * Arguments are as for fa_decode_paged; sizes whose
 * fa_decode_workspace_size(S, H, d, max_blocks_per_seq) exceeds FA_NOALLOC_SCRATCH_BYTES return
 * FA_ERR_WORKSPACE (fa_last_error_string() says how many bytes were needed) and launch nothing.
 * No slot of the array needs to start at zero: every slot a call reads was written earlier in
 * that same call.  All calls share the one array, so two calls that overlap on the GPU (other
 * streams, other host threads) race and corrupt each other's results: serialise them.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

fa_status fa_decode_paged_noalloc(const void *q, const void *k_pool, const void *v_pool,
                                  const int32_t *block_table, int max_blocks_per_seq,
                                  const int32_t *seq_lens, int num_blocks, void *o,
                                  fa_out_dtype o_dtype, float *lse, int S, int H, int d,
                                  float scale, fa_stream_t stream);

/*
 * fa_get_device_status -- synchronises `stream`, then reads and clears the library's device
 * status word.  Returns FA_OK, FA_ERR_TIMEOUT (a kernel abandoned a wait), or FA_ERR_LAUNCH if the
 * synchronisation itself reported a CUDA error.
 */
fa_status fa_get_device_status(fa_stream_t stream);

/*
 * fa_selftest_wait_timeout -- diagnostic: launches one thread that waits on a barrier nothing ever
 * signals, through the same bounded wait the attention kernels use, with a limit of `limit_us`
 * microseconds (1 .. 2000000).  The wait gives up, the kernel records FA_ERR_TIMEOUT in the device
 * status word and returns, and the context stays usable.  Lets a caller (or a test) confirm that
 * a stalled kernel is reported through fa_get_device_status instead of hanging the GPU.
 */
fa_status fa_selftest_wait_timeout(unsigned limit_us, fa_stream_t stream);

/*
 * fa_probe_ex2_rate -- diagnostic: launches a kernel (4 CTAs of 256 threads per SM) whose threads
 * each evaluate `iters` x 16 base-2 exponentials on the special-function unit, the instruction the
 * online softmax uses for p = 2^(s * scale * log2 e - m) ("Flash Attention" (myungum), section 2,
 * the exponentials of each score block).  Writes the number of exponentials launched to *exps_out
 * (host memory); the caller times the launch on `stream` and divides.  The result is the ceiling
 * that the exponentials put on the forward: one per 4 d FLOP of Q K^T and P V.  `sink` is one
 * float of device memory the kernel may write (it never does for these inputs).  iters in
 * 1 .. 2^24, else FA_ERR_INVALID_ARG.
 */
fa_status fa_probe_ex2_rate(float *sink, int iters, long long *exps_out, fa_stream_t stream);

/*
 * fa_probe_read_rate -- diagnostic: reads `bytes` (a multiple of 16, >= 16) of device memory at
 * `buf` (16-byte aligned) once, with the 16-byte streaming loads the paged decode uses to walk the
 * KV cache ("LLM study notes", paged attention: decode reads every cached key and value), from
 * 4 CTAs of 512 threads per SM.  The caller times the launch on `stream`: bytes / time is the
 * read-only HBM bandwidth that bounds the decode, which only reads.  `sink` is one float of device
 * memory the kernel may write.  Bad sizes or pointers return FA_ERR_INVALID_ARG /
 * FA_ERR_ALIGNMENT before anything launches.
 */
fa_status fa_probe_read_rate(const void *buf, size_t bytes, float *sink, fa_stream_t stream);

/*
 * fa_fwd_schedule -- host only: the assignment of work units to CTAs that a causal fa_fwd launch
 * of this shape makes on a GPU with num_ctas SMs; no device is touched.  Work is split over batch,
 * head and query tile ("FlashAttention-2 GPU work partitioning", section 3): a unit is one pair of
 * 128-row query tiles of one (b, h), numbered level-major, so unit u covers (b*H + h) = u % (B*H)
 * and query tiles 2p and 2p + 1 with p = ceil(N / 256) - 1 - u / (B*H); its cost grows with p.
 * At d = 128 the launch balances the CTAs by list scheduling over heads taken in groups whose K and
 * V fill a fraction of L2, longest units first within a group, so that one group's K and V stay
 * resident; at d = 64 (bound by its exponentials, not by DRAM) it always deals in snake order.
 *
 *   B, H, N, d  as for fa_fwd (d: 64 or 128);  num_ctas in 1 .. 1024.
 *   start       int [num_ctas + 1], host memory: CTA c runs unit[start[c]] .. unit[start[c+1] - 1]
 *               in that order.  Entries past the launch's CTA count G = min(units, num_ctas) are
 *               set to the unit count.
 *   unit        int [capacity], host memory.
 *   *count      the number of units in the table, or 0 when the launch takes no table: it then
 *               deals the units in snake order (round r gives CTA c unit r*G + c for even r and
 *               r*G + G-1-c for odd r), and start / unit are not written.
 * FA_ERR_INVALID_ARG for bad sizes, null pointers, or a capacity below the unit count.
 */
fa_status fa_fwd_schedule(int B, int H, int N, int d, int num_ctas, int *start, int *unit,
                          int capacity, int *count);

/* Static text for a status code. */
const char *fa_status_string(fa_status status);

/* The CUDA error text of the last FA_ERR_LAUNCH on this thread, or the scratch size that
 * fa_decode_paged_noalloc needed when it returned FA_ERR_WORKSPACE ("" if none). */
const char *fa_last_error_string(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
