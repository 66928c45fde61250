/*
 * kda_prefill.h -- C ABI of the KDA (Kimi Delta Attention) chunk-prefill
 * forward for NVIDIA B200 (sm_100a).
 *
 * The operation ("KDA Chunk Prefill on Ascend A3", sections "Function and
 * tensor contract" and "Mathematical definition"):
 *
 *   forward(q, k, v, g, beta, initial_state) -> (o, final_state)
 *
 *   1. Q and K are L2-normalised along their last dimension in float32 in
 *      the stated rounding order, epsilon 1e-6 inside the square root, and
 *      rounded to bf16:  xn = bf16(f32(x) / sqrt(sum(f32(x)^2) + 1e-6)).
 *   2. For every sequence and value head h (Q/K head h / (HV/H)), with a
 *      float32 state S[K][V], the gated delta rule runs over the tokens:
 *         S   <- exp(g_t)[:,None] * S
 *         r_t  = v_t - k_t^T S
 *         S   <- S + beta_t k_t r_t^T
 *         o_t  = (K^-0.5 q_t)^T S
 *      The library evaluates it in the page's chunk form (64-token chunks:
 *      cumulative gate G, strictly lower L, causal Aqk, A = (I+L)^-1
 *      diag(beta), W = A (exp(G) k), U = A v, and the inter-chunk carry
 *      Vnew = U - W S, O = Qg S + Aqk Vnew, S' = exp(G_last) S + Kg^T Vnew).
 *      A partial last chunk behaves as if zero-padded; its padded rows are
 *      never written.
 *
 * Conventions shared by every entry point:
 *   - All tensors are dense, row-major (C order), contiguous.  Pointers are
 *     caller-owned DEVICE memory unless the name says _host.  The library
 *     never allocates device memory and never synchronises the stream.
 *   - Inputs are never written.  final_state may alias initial_state
 *     exactly (in-place update); any other overlap is rejected.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Argument errors are detected on the host before any
 *     launch; launch failures are reported as KDA_ERR_CUDA.  Values held in
 *     device memory (cu_seqlens entries) are not checked on the host.
 *   - Supported sizes: K == V == 128, HV % H == 0, all sizes positive
 *     (T may be 0 only with cu_seqlens).  Other K/V give
 *     KDA_ERR_UNSUPPORTED.
 *   - Numerical domain: gates g <= 0 with sum over any 16 consecutive
 *     tokens >= -80 (per-token g >= -5 suffices); beta in [0, 1]; |v| and
 *     the state entries below 6e4 (the state-carry contractions use fp16
 *     operands with fp32 accumulation; the gate-rescaled L/Aqk operands use
 *     bf16 for its range).
 */
#ifndef KDA_PREFILL_H
#define KDA_PREFILL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, HV % H != 0, bad overlap */
    KDA_ERR_UNSUPPORTED = 2, /* K or V other than 128 */
    KDA_ERR_MISALIGNED = 3,  /* a pointer is not aligned as documented */
    KDA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than kda_prefill_workspace_size() */
    KDA_ERR_CUDA = 5         /* a CUDA runtime call or a kernel launch failed */
} kda_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status_t status);

/*
 * Bytes of device workspace kda_prefill_forward needs for these sizes.
 * num_seqs is the number of packed sequences when cu_seqlens is used, or 0
 * for a plain [B, T] batch.  The workspace holds, per (64-token chunk, value
 * head), the chunk's state-independent results that the intra-chunk kernel
 * hands to the carry kernel (72.5 KiB each), plus the chunk offsets, the
 * longest-first order and the chunk-window offsets (4 x (N + 1) int32) of
 * packed sequences, and, for plain batches of few long
 * sequences, room for the segmented carry's states (3 x B x HV x S x 64 KiB,
 * S as described at kda_prefill_forward).  Returns 0 for sizes that
 * kda_prefill_forward would reject.
 */
size_t kda_prefill_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs);

/*
 * The chunk-prefill forward.
 *
 *   q, k          bf16 [B, T, H, K]        16-byte aligned
 *   v             bf16 [B, T, HV, V]       16-byte aligned
 *   g             fp32 [B, T, HV, K]       16-byte aligned; natural-log gates
 *   beta          fp32 [B, T, HV]          4-byte aligned
 *   initial_state fp32 [N, HV, K, V] or NULL (zeros); 4-byte aligned
 *   cu_seqlens    int32 [N + 1] or NULL.   When given: B == 1, N = num_seqs >= 1,
 *                 cu_seqlens[0] == 0, non-decreasing, cu_seqlens[N] == T
 *                 (device values, not checked).  Sequence n holds tokens
 *                 [cu[n], cu[n+1]) and starts from initial_state[n].
 *                 When NULL: N = B and num_seqs is ignored.
 *   o             bf16 [B, T, HV, V] out;  16-byte aligned.  Rows of tokens
 *                 that belong to no sequence are left untouched.
 *   final_state   fp32 [N, HV, K, V] out (required); 4-byte aligned
 *   workspace     device scratch of at least kda_prefill_workspace_size()
 *                 bytes, 256-byte aligned, overlapping no other argument.
 *                 Its contents need no initialisation and are garbage after.
 *   stream        cudaStream_t
 *
 * Asynchronous on `stream`.  A plain batch (cu_seqlens NULL) with fewer
 * (sequence, value head) pairs than the device has SMs and at least 32
 * chunks per sequence is run as up to 8 consecutive parts of the sequence
 * (whole chunks): the state carry of each part runs on a high-priority side
 * stream of the library, overlapping the intra-chunk work of the next part,
 * and joins `stream` again through an event before the call returns, so the
 * caller sees one ordered operation (under stream capture the side stream
 * becomes a fork and join of the captured graph).  The library keeps four
 * such side streams per device and a call takes a free one, so calls that
 * host threads make at the same time get different side streams (a fifth
 * concurrent call waits on the host for the first to finish enqueueing).
 *
 * A plain batch with few units (B * HV <= 48) and long sequences may
 * instead carry S segments of every sequence at once: the segments' linear
 * maps and images of zero, a scan of their start states, then all segments
 * with outputs (4 launches in all, on `stream`).  The workspace reserves
 * room for S up to min(1024 / (2 B HV + 1), ceil(T/64) / 16); the forward
 * picks S on the device when its cost model says the segments are faster
 * than the overlapped carry.  The results follow the same recurrence with a
 * different rounding order.
 */
kda_status_t kda_prefill_forward(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 const float *initial_state,
                                 const int32_t *cu_seqlens, int num_seqs,
                                 int B, int T, int H, int HV, int K, int V,
                                 void *o, float *final_state,
                                 void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * kda_prefill_forward on a packed batch whose sequence boundaries the caller
 * also holds on the host (the page's packed-sequence contract, "Function and
 * tensor contract": sequence n is tokens [cu[n], cu[n+1]) with its own
 * state).  Same arguments as kda_prefill_forward with B = 1, plus:
 *   cu_seqlens_host  int32 [num_seqs + 1] in host memory holding the same
 *                    values as cu_seqlens; read during the call only.  It
 *                    must start at 0, end at T and not decrease, else
 *                    KDA_ERR_INVALID_ARG.
 * Knowing the lengths, the library can overlap the state carry with the
 * intra-chunk work.  This happens when the longest sequence has at least 32
 * chunks, and the (sequence, value head) pairs of the sequences longer than
 * the first window are fewer than the device's SMs.  The batch is then cut
 * into up to 4 windows of chunk index within each sequence (the longest
 * sequence's chunks in equal windows but the last, which is a quarter of
 * the others).  The state carry of window j (every sequence with chunks in
 * it, longest first) runs beside the intra-chunk work of window j+1: that
 * intra-chunk kernel is a programmatic dependent launch of the carry, which
 * lets it start once every carry CTA is resident.  Everything stays on
 * `stream`.  Otherwise the call runs exactly as kda_prefill_forward.  Either
 * way the results are bit-identical to kda_prefill_forward's.  Workspace:
 * kda_prefill_workspace_size(1, T, H, HV, K, V, num_seqs).
 */
kda_status_t kda_prefill_forward_varlen(const void *q, const void *k, const void *v,
                                        const float *g, const float *beta,
                                        const float *initial_state,
                                        const int32_t *cu_seqlens,
                                        const int32_t *cu_seqlens_host, int num_seqs,
                                        int T, int H, int HV, int K, int V,
                                        void *o, float *final_state,
                                        void *workspace, size_t workspace_bytes,
                                        void *stream);

/*
 * Kernel launches kda_prefill_forward_varlen makes for these lengths on the
 * current device (0 if it would reject them).
 */
int kda_prefill_varlen_kernel_launches(int T, int H, int HV, int K, int V, int num_seqs,
                                       const int32_t *cu_seqlens_host);

/*
 * Bytes of device staging memory kda_prefill_forward_host needs: room for
 * every input and output plus the workspace, each 256-byte aligned.
 */
size_t kda_prefill_host_staging_size(int B, int T, int H, int HV, int K, int V, int num_seqs,
                                     int has_initial_state, int has_cu_seqlens);

/*
 * The same forward on HOST buffers (same shapes and dtypes as above; pinned
 * memory makes the copies asynchronous).  Inputs are copied into the
 * caller's device staging buffer, the forward runs there, and o and
 * final_state are copied back -- all ordered after `stream`'s earlier work
 * and before its later work; the caller synchronises before reading
 * o_host / final_state_host.  Where the forward cuts a plain batch into
 * parts (see kda_prefill_kernel_launches), each part's input rows are
 * uploaded on a copy stream of the library while the earlier parts compute,
 * and each part's o rows are downloaded as soon as its carry has run, so
 * the two copy directions overlap; the results equal kda_prefill_forward's
 * bit for bit.  A packed batch runs through kda_prefill_forward_varlen with
 * cu_seqlens_host as its host copy of the boundaries, so its carry can
 * overlap the intra-chunk work (its copies are not split).  Calls on one device are serialised by the library while
 * they enqueue (the copy streams are shared).
 */
kda_status_t kda_prefill_forward_host(const void *q_host, const void *k_host, const void *v_host,
                                      const float *g_host, const float *beta_host,
                                      const float *initial_state_host,
                                      const int32_t *cu_seqlens_host, int num_seqs,
                                      int B, int T, int H, int HV, int K, int V,
                                      void *o_host, float *final_state_host,
                                      void *staging, size_t staging_bytes,
                                      void *stream);

/*
 * kda_prefill_forward without a workspace argument, for callers that cannot
 * allocate device memory: runtimes that freeze their device memory after
 * warm-up (cudaMalloc synchronises the whole device and would stall every
 * other stream) and plugin hosts that give plugins no allocator.  The page
 * has no counterpart of this entry point; it is a packaging choice.
 *
 * Same arguments and behaviour as kda_prefill_forward minus workspace /
 * workspace_bytes.  The workspace is a fixed 64 MiB device array that every
 * GPU loading the library reserves until the process exits; sizes whose
 * kda_prefill_workspace_size() exceeds 64 MiB (about 900 pairs of a 64-token
 * chunk and a value head, e.g. T = 14,400 at HV = 4) are rejected with
 * KDA_ERR_WORKSPACE before any launch.  The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  The address is kept for the life of the
 * process: after cudaDeviceReset (or anything else that destroys the
 * device's primary context) it is stale, so do not call this entry point on
 * that device again in the same process.  Every call shares the one array, so calls
 * whose work overlaps on the GPU (other streams, other threads) race; issue
 * them one after another.  Calls no cudaMalloc / cudaFree.
 */
kda_status_t kda_prefill_forward_noalloc(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta,
                                         const float *initial_state,
                                         const int32_t *cu_seqlens, int num_seqs,
                                         int B, int T, int H, int HV, int K, int V,
                                         void *o, float *final_state, void *stream);

/*
 * Debug aid: the device error word of the current device.  Kernel waits on
 * copies and pipeline stages are bounded (about one second); a wait that
 * gives up sets a bit here (1: input tile copy, 2: stage fill, 4: stage
 * release) and the kernel stops early instead of hanging; bit 8 means a
 * tensor-memory allocation did not start at column 0 (not expected to happen).  Synchronises the
 * device.  clear != 0 resets the word afterwards.
 */
kda_status_t kda_prefill_device_error(unsigned *word, int clear);

/*
 * Number of kernel launches kda_prefill_forward makes for these sizes on the
 * current device (the split into parts above depends on its SM count), or 0
 * for sizes it would reject.
 */
int kda_prefill_kernel_launches(int B, int T, int H, int HV, int K, int V, int num_seqs);

/*
 * The forward with the state stored in bf16 (a precision variant the pages
 * allow: "KDA Chunk Prefill on Ascend A3", section "Function and tensor
 * contract", leaves the state's storage open beyond fp32 results): arguments
 * as kda_prefill_forward except
 *   initial_state  bf16 [N,HV,K,V] or NULL, 16-byte aligned
 *   final_state    bf16 [N,HV,K,V] out (nearest-even rounding of the fp32
 *                  state the forward computes); may equal initial_state
 *   workspace      kda_prefill_state_bf16_workspace_size(...) bytes
 * The state is widened to fp32 before the carry and rounded after it; the
 * arithmetic in between is the fp32-state forward's.
 */
size_t kda_prefill_state_bf16_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs);
kda_status_t kda_prefill_forward_state_bf16(const void *q, const void *k, const void *v, const float *g,
                                            const float *beta, const void *initial_state, const int32_t *cu_seqlens,
                                            int num_seqs, int B, int T, int H, int HV, int K, int V, void *o,
                                            void *final_state, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward of kda_prefill_forward, which "KDA Chunk Prefill on Ascend A3"
 * leaves optional (section "Timing and required submission"): for the loss
 * sum(o * dout) + sum(final_state * dht) it returns the gradients of q, k,
 * v, g, beta and the initial state in their own dtypes.  The bf16 rounding
 * of the normalised q/k rows is passed straight through (its derivative is
 * taken as one): dq = J(q)^T sum_h dqn_h, J the Jacobian of
 * q / sqrt(sum q^2 + 1e-6) and the sum over the value heads h that read q.
 *
 *   q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, B, T, H, HV, K, V
 *                as for kda_prefill_forward (initial_state may be NULL)
 *   dout         bf16 [B,T,HV,V]   gradient of the loss at o
 *   dht          fp32 [N,HV,K,V]   gradient at final_state, or NULL (zero)
 *   dq, dk       bf16 [B,T,H,K]    out
 *   dv           bf16 [B,T,HV,V]   out
 *   dg           fp32 [B,T,HV,K]   out
 *   dbeta        fp32 [B,T,HV]     out
 *   dh0          fp32 [N,HV,K,V]   out, or NULL when not wanted
 *   workspace    kda_prefill_backward_workspace_size(...) bytes, 256-byte
 *                aligned, device; holds the recomputed forward's per-chunk
 *                blocks, every chunk's start state and the gradient at every
 *                chunk's end state (bf16), and per-value-head gradients at the
 *                normalised rows (fp32).
 * Outputs overlap no input, no other output and the workspace.  Pointers are
 * 16-byte aligned (beta, dbeta, cu_seqlens: 4).  Rows outside every packed
 * sequence are left untouched.  Asynchronous on `stream`; kernel waits that
 * give up set the device error word (kda_prefill_device_error).
 *
 * The forward is recomputed (intra-chunk blocks, then the state carry storing
 * each chunk's start state; a long sequence is cut into parts as the forward
 * cuts it, each part's carry beside the next part's blocks); a reverse carry
 * walks each sequence backwards
 * for the gradient at every chunk's end state; a per-chunk kernel forms the
 * chunk's gradients (and, when H == HV, applies the normalisation's
 * Jacobian); with H < HV a last kernel sums each Q/K group and applies it.
 * Accuracy assumes g <= 0 with every 8 consecutive gates of a channel summing
 * to >= -40 (per-token g >= -5 suffices), and, as for the forward's state,
 * entries of the chunk states, of their gradients and of dout below 6e4: the
 * reverse carry and the per-chunk passes multiply them as fp16 operands.
 */
size_t kda_prefill_backward_workspace_size(int B, int T, int H, int HV, int K, int V, int num_seqs);
/* Kernel launches of one kda_prefill_backward call (the recomputing form); 0 for invalid sizes, or when the
 * sizes are long enough to be cut into parts and the current device cannot be queried. */
int kda_prefill_backward_kernel_launches(int B, int T, int H, int HV, int K, int V, int num_seqs);
kda_status_t kda_prefill_backward(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                  const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B,
                                  int T, int H, int HV, int K, int V, const void *dout, const float *dht, void *dq,
                                  void *dk, void *dv, float *dg, float *dbeta, float *dh0, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * The forward that keeps what the backward needs, and the backward from it
 * (the usual save-for-backward split of a training step):
 *   kda_prefill_forward_save   the forward (arguments as kda_prefill_forward)
 *                              that also leaves its per-chunk blocks and
 *                              every chunk's start state (bf16) in `saved`;
 *   kda_prefill_backward_saved the backward (arguments as kda_prefill_backward)
 *                              with `saved` as its workspace; it skips the
 *                              forward's recomputation.
 * `saved` is kda_prefill_backward_workspace_size(...) bytes, 256-byte aligned,
 * device, overlapping no argument; it must reach the backward unchanged and the
 * backward must get the same q, k, v, g, beta, initial_state and cu_seqlens.
 */
kda_status_t kda_prefill_forward_save(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                      const float *initial_state, const int32_t *cu_seqlens, int num_seqs, int B,
                                      int T, int H, int HV, int K, int V, void *o, float *final_state, void *saved,
                                      size_t saved_bytes, void *stream);
kda_status_t kda_prefill_backward_saved(const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                                        int num_seqs, int B, int T, int H, int HV, int K, int V, const void *dout,
                                        const float *dht, void *dq, void *dk, void *dv, float *dg, float *dbeta,
                                        float *dh0, void *saved, size_t saved_bytes, void *stream);

/*
 * One recurrent decode step (one token per row) on a caller-owned bf16 state
 * pool, as on the "flashinfer.kda_decode.packed_kda_decode" page, with the
 * recurrence of "KDA Chunk Prefill on Ascend A3" (section "Mathematical
 * definition") for T = 1.  The page's gate and beta activations (its
 * lower-bound gate formula is not given there) are the caller's: g and beta
 * arrive activated, as in kda_prefill_forward.
 *
 *   q, k          bf16, row b at q + b * q_row_stride: [H, K]; rows 8-byte
 *                 aligned, strides multiples of 4 elements (a packed QKV row
 *                 [q | k | v] is passed as three pointers with one stride)
 *   v             bf16, row b at v + b * v_row_stride: [HV, V]
 *   g             fp32 [B, HV, K]  natural-log gates, <= 0
 *   beta          fp32 [B, HV]
 *   state         bf16 pool of num_slots slots; slot s at state +
 *                 s * slot_stride elements holds [HV, K, V] (compact inside;
 *                 slot_stride >= HV*K*V, a multiple of 8); 16-byte aligned.
 *                 Updated in place: slot <- bf16 (nearest even) of the new
 *                 state computed in fp32.
 *   state_indices int32 [B] device: the slot of each row, or -1 for a padding
 *                 row, whose output is zeros and which touches no state.
 *                 Active indices must be unique and < num_slots (device
 *                 values, not checked).
 *   o             bf16 [B, HV, V] out, overlapping no other argument.
 * B = 0 is a no-op.  K = V = 128.  Asynchronous on `stream`.  Each (row,
 * value head) state block moves by bulk copy through shared memory; a copy
 * that has not landed after about a second sets bit 1 of the device error
 * word (kda_prefill_device_error) and the kernel stops.
 */
kda_status_t kda_decode_step(const void *q, int64_t q_row_stride, const void *k, int64_t k_row_stride,
                             const void *v, int64_t v_row_stride, const float *g, const float *beta,
                             void *state, int64_t slot_stride, int num_slots, const int32_t *state_indices,
                             int B, int H, int HV, int K, int V, void *o, void *stream);

/*
 * Step 1 alone: L2-normalise `rows` rows of K bf16 values with the exact
 * rounding order above ("KDA Chunk Prefill on Ascend A3", section
 * "Mathematical definition", first formula).  x and out: bf16 [rows, K],
 * 16-byte aligned, device; out may equal x.  K must be 128.
 */
kda_status_t kda_l2norm_bf16(const void *x, int64_t rows, int K, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_PREFILL_H */
