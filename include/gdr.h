/*
 * gdr.h -- C ABI of the gated delta-rule layer library (libgdr.so), sm_100a.
 *
 * The layer (one of the 54 recurrent layers of the hybrid decoder described in
 * "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型", section 注意力层的细节):
 * 16 key heads and 48 value heads of dimension 128, a kernel-4 depthwise
 * causal conv with SiLU in front, L2-normalised q and k, a decay gate and a
 * write strength per token and value head, an fp32 recurrent state of
 * 128 x 128 per value head, and a gated RMSNorm on the output.
 *
 * The recurrence ("Sapiens AI 发布 Agnes-3.0-Flash", section
 * "delta 规则循环层究竟怎么运作", with the forget gate of the gated variant):
 *     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 * with ("33B 只做 18 层：Agnes 3.0 Flash ...", §1.2)
 *     beta_t = sigmoid(b_t),  g_t = -exp(A_log) * softplus(a_t + dt_bias)
 * computed in fp32, and q, k divided by sqrt(sum x^2 + 1e-6) inside the
 * kernels.  Value head h reads key head h / (hv / hk).
 *
 * Conventions shared by every entry point
 *  - Tensor pointers are DEVICE memory owned by the caller, except the
 *    `*_host` arguments, which are host memory.  The library allocates no
 *    device memory and keeps no per-call state; it writes a device-side error
 *    word only when a kernel hits a bounded wait (gdr_get_device_error).
 *  - bf16 tensors are passed as `void *` holding IEEE bfloat16 values; fp32
 *    tensors as `float *`.  All layouts are dense row-major (C order) with the
 *    shapes written next to each argument.  Every tensor pointer must be
 *    16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously; no call synchronises the device.
 *  - Kernels are launched with programmatic dependent launch: each may be
 *    scheduled while the work before it on the stream drains, but waits for
 *    that work to complete (griddepcontrol.wait) before it reads or writes any
 *    memory, so stream order is kept.  A caller's kernel that follows on the
 *    stream and is itself launched with programmatic stream serialization
 *    must wait the same way (cudaGridDependencySynchronize) before it reads
 *    this library's outputs; one launched without it is simply ordered.
 *  - The recurrent state is stored transposed, H = S^T, as
 *    [n][hv][dk][dv] fp32 (the dv index is contiguous).
 *  - Supported dims: dk = dv = 128, hk >= 1, hv % hk == 0, hv / hk <= 8.
 *  - A non-zero return value is a gdr_status_t; nothing has been launched
 *    when an argument check fails.  GDR_ERR_CUDA reports a failed launch.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdr_status {
  GDR_OK = 0,
  GDR_ERR_NULL = 1,        /* a required pointer is NULL */
  GDR_ERR_SHAPE = 2,       /* a size is negative, zero where it must not be, or inconsistent */
  GDR_ERR_ALIGN = 3,       /* a tensor pointer is not 16-byte aligned */
  GDR_ERR_CU_SEQLENS = 4,  /* cu_seqlens does not start at 0 or decreases */
  GDR_ERR_UNSUPPORTED = 5, /* head dims / grouping outside what the kernels implement */
  GDR_ERR_WORKSPACE = 6,   /* the prefill workspace is NULL or too small for one chunk window */
  GDR_ERR_CUDA = 7,        /* the CUDA launch failed (see cudaGetLastError) */
  GDR_ERR_TIMEOUT = 8,     /* (device error word) a bounded wait inside a kernel ran out */
  GDR_ERR_ALIAS = 9        /* two buffers overlap where the call forbids it */
} gdr_status_t;

/* Human-readable name of a status code.  Never NULL. */
GDR_API const char *gdr_status_string(int status);

/* ABI version of this header, bumped whenever a signature or what a call does
 * changes (2: the conv fused into gdr_chunk_prefill,
 * gdr_chunk_prefill_fused_workspace_size; 3: gdr_decode_step_slots; 4:
 * gdr_chunk_prefill_slots; 5: gdr_chunk_prefill_schedule and the
 * pipelined window schedule; 6: gdr_linear). */
GDR_API int gdr_abi_version(void);

/*
 * Chunk table of packed sequences (host only, no device work).
 * Chunks of `chunk` tokens restart at every sequence start; the last chunk of
 * a sequence may be shorter; empty sequences have no chunk.  Chunks are listed
 * sequence by sequence in token order: chunk m covers tokens
 * [chunk_start[m], chunk_start[m] + chunk_len[m]) of sequence chunk_seq[m].
 *   cu_seqlens_host: [n_seqs + 1] int32 token offsets, cu[0] = 0, non-decreasing.
 *   chunk_seq, chunk_start, chunk_len: host arrays of max_chunks entries.
 * Returns GDR_ERR_CU_SEQLENS for an invalid offset array and GDR_ERR_SHAPE if
 * the table needs more than max_chunks entries; *n_chunks receives the count.
 * The prefill kernel walks exactly this table.
 */
GDR_API int gdr_prepare_chunks(const int32_t *cu_seqlens_host, int n_seqs, int chunk, int32_t *chunk_seq,
                       int32_t *chunk_start, int32_t *chunk_len, int max_chunks, int *n_chunks);

/*
 * gdr_causal_conv -- depthwise causal conv, kernel 4, followed by SiLU,
 * over packed sequences ("Agnes-3.0-Flash 深度解析", 注意力层的细节: a kernel-4
 * causal conv in front of the recurrence).
 *     y[t][c] = SiLU(sum_{j=0..3} w[c][j] * x[t-3+j][c])   (fp32 math, bf16 out)
 * w[c][3] multiplies the current token.  Inputs before a sequence's first
 * token come from conv_state_in[n] (oldest first) or are zero when
 * conv_state_in is NULL; nothing crosses a cu_seqlens boundary.
 *   x:              bf16 [T][channels]        (T = cu_seqlens_host[n_seqs])
 *   w:              bf16 [channels][4]
 *   conv_state_in:  bf16 [n_seqs][3][channels] or NULL
 *   conv_state_out: bf16 [n_seqs][3][channels] or NULL; receives the last three
 *                   inputs of each sequence (shifted from conv_state_in when a
 *                   sequence is shorter than three).  Must not overlap
 *                   conv_state_in (GDR_ERR_ALIAS).
 *   cu_seqlens_dev / cu_seqlens_host: the same [n_seqs + 1] int32 offsets on
 *                   the device and on the host.
 *   y:              bf16 [T][channels]; channels % 8 == 0.
 */
GDR_API int gdr_causal_conv(const void *x, const void *w, const void *conv_state_in, void *conv_state_out,
                    const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seqs,
                    int channels, void *y, void *stream);

/*
 * Optional work around the prefill (pass NULL to gdr_chunk_prefill to run
 * the recurrence alone).
 *  - Gated RMSNorm (`z` set), a fusion: y receives o / sqrt(mean(o^2) + eps) *
 *    w * SiLU(z) row by row, computed from the bf16-rounded o inside the
 *    prefill's state kernel (the two 64-column halves of a head run as a
 *    thread-block cluster and exchange their row sums of squares), so o need not
 *    go through memory; o is written as well only when gdr_chunk_prefill's o is
 *    not NULL.  y must not overlap o (GDR_ERR_ALIAS).  It saves the o round
 *    trip but lengthens the state kernel's per-chunk path, and at one sequence
 *    it runs slower than the separate gdr_gated_rmsnorm call.
 *  - Conv (`x` set), a convenience, not a fusion: the call runs the kernel of
 *    gdr_causal_conv on x (with conv_w and the optional conv states) into the
 *    head of the workspace and the prefill reads q, k, v from there, so the
 *    caller needs no conv output buffer.  The conv output is still written to
 *    and read back from device memory: the bytes moved are those of the two
 *    separate calls.  q, k and v must then be NULL (GDR_ERR_SHAPE otherwise)
 *    and the workspace must hold gdr_chunk_prefill_fused_workspace_size(...)
 *    bytes.  conv_state_out receives the last three inputs of every sequence
 *    (empty ones included), as from gdr_causal_conv.  The results equal the
 *    separate calls bit for bit: the same kernels run, one after the other on
 *    the stream.
 */
typedef struct gdr_prefill_fuse {
  const void *x;             /* bf16 [T][hk*128*2 + hv*128] conv input, or NULL */
  const void *conv_w;        /* bf16 [channels][4] (required with x) */
  const void *conv_state_in; /* bf16 [n_seqs][3][channels] or NULL (zeros) */
  void *conv_state_out;      /* bf16 [n_seqs][3][channels] or NULL; must not overlap conv_state_in */
  const void *z;             /* bf16 [T][hv][128] gate of the RMSNorm, or NULL */
  const float *norm_w;       /* fp32 [128] norm weight, or NULL (ones) */
  float eps;                 /* RMSNorm epsilon */
  void *y;                   /* bf16 [T][hv][128] (required with z) */
} gdr_prefill_fuse_t;

/*
 * gdr_chunk_prefill -- the recurrence over packed sequences, chunk of 64
 * ("33B 只做 18 层 ...", §1.2: prefill takes the chunk-64 path, said to be
 * interchangeable with the per-token one).
 * Per chunk the kernel uses the WY/UT form of the unrolled recurrence; the
 * dense products run on the tcgen05 tensor cores and the state carried from
 * chunk to chunk stays fp32.
 *   q, k:     bf16 [T][hk][128] rows, consecutive tokens qk_token_stride
 *             elements apart (0 = dense, hk*128); NULL (with v) when the conv
 *             is fused (fuse->x), the strides are then ignored
 *   v:        bf16 [T][hv][128] rows, consecutive tokens v_token_stride
 *             elements apart (0 = dense, hv*128).  The strides let q, k, v be
 *             read in place from the [T][q | k | v] conv output (stride
 *             2*hk*128 + hv*128); a stride must be a multiple of 8.
 *   a, b:     bf16 [T][hv]            gate inputs (see the header comment)
 *   A_log, dt_bias: fp32 [hv]
 *   scale:    output scale
 *   cu_seqlens_dev / cu_seqlens_host: [n_seqs + 1] int32, same values.
 *   h0:       fp32 [n_seqs][hv][128][128] initial state (H = S^T), or NULL = zeros
 *   hT:       fp32 [n_seqs][hv][128][128] final state, or NULL; may equal h0
 *             (in place), must not overlap it otherwise.
 *   o:        bf16 [T][hv][128]; may be NULL when fuse->y is set (fused norm).
 *   fuse:     NULL, or conv / gated-norm fusion (see gdr_prefill_fuse_t).
 *   workspace, workspace_bytes: device scratch, 16-byte aligned, at least
 *             gdr_chunk_prefill_workspace_size(n_seqs, hv, 1, hT != NULL)
 *             bytes (GDR_ERR_WORKSPACE otherwise); the window is the largest
 *             number of chunks that fits.
 * Empty sequences copy h0 (or zeros) to hT.
 * Long sequences on a GPU that the state kernels leave partly idle (n_seqs *
 * hv * 2 below the SM count, e.g. one sequence of 48 value heads): when the
 * workspace holds two windows of at least 16 chunks and the sequences need at
 * least three such windows, the call splits the workspace into two record
 * buffers and builds window w + 1 while window w's state walk runs, on a pair
 * of streams the library creates once per device (high and low priority).
 * The work forks from `stream` and joins it before the call returns; the
 * results equal the one-buffer schedule bit for bit.  Calls that pipeline on
 * one device take turns issuing (a lock).  A call made while `stream` is
 * being captured into a graph keeps the one-buffer schedule on `stream`.
 */
GDR_API int gdr_chunk_prefill(const void *q, const void *k, const void *v, int64_t qk_token_stride,
                              int64_t v_token_stride, const void *a, const void *b,
                              const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                              const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                              int n_seqs, const float *h0, float *hT, void *o,
                              const gdr_prefill_fuse_t *fuse, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Bytes of device workspace gdr_chunk_prefill needs to build the
 * state-independent operands of `window_chunks` chunks of every sequence at a
 * time (81 KiB per sequence, value head and chunk), plus room to carry the
 * state between windows when hT is NULL (has_final_state == 0).  Any
 * window_chunks >= 1 is valid; a window of ceil(max sequence length / 64)
 * chunks processes everything in one pass, smaller windows use less memory
 * and more kernel launches.  The workspace is caller-owned scratch: its
 * contents need no initialisation and are meaningless after the call, and
 * two calls in flight at the same time must not share it.
 */
GDR_API size_t gdr_chunk_prefill_workspace_size(int n_seqs, int hv, int window_chunks,
                                                int has_final_state);

/*
 * The window schedule gdr_chunk_prefill (and gdr_chunk_prefill_slots,
 * has_final_state = 0) follows for these sequences and this workspace on the
 * current device, outside stream capture: *windows receives the number of
 * windows (each one launch of the operand kernel and one of the state kernel;
 * 1 when no sequence has a token) and *pipelined 1 when window w + 1 is built
 * beside window w's state walk (the two-buffer schedule described under
 * gdr_chunk_prefill), else 0.  Host only; it may query the device's SM
 * count.  Returns GDR_ERR_NULL for a NULL pointer, GDR_ERR_SHAPE for hv <= 0,
 * a negative n_seqs or has_final_state not 0 or 1, GDR_ERR_CU_SEQLENS for
 * bad offsets, GDR_ERR_WORKSPACE when not one chunk of every sequence fits.
 */
GDR_API int gdr_chunk_prefill_schedule(const int32_t *cu_seqlens_host, int n_seqs, int hv,
                                       size_t workspace_bytes, int has_final_state, int *windows,
                                       int *pipelined);

/*
 * Bytes of device workspace gdr_chunk_prefill needs with the conv fused
 * (gdr_prefill_fuse_t.x set): the conv output of the total_tokens tokens,
 * [total_tokens][hk*128*2 + hv*128] bf16 rounded up to a whole KiB, followed by
 * gdr_chunk_prefill_workspace_size(n_seqs, hv, window_chunks, has_final_state).
 * Returns 0 for invalid sizes.
 */
GDR_API size_t gdr_chunk_prefill_fused_workspace_size(int n_seqs, int hk, int hv, int total_tokens,
                                                      int window_chunks, int has_final_state);

/*
 * gdr_chunk_prefill_noalloc -- gdr_chunk_prefill without a caller workspace.
 * (No counterpart in the pages that describe the layer: this is an interface
 * convenience of this library.)
 * For callers that cannot allocate device memory: a plugin whose host
 * framework owns all device memory and hands out no scratch buffers, a
 * fixed-budget deployment that must not grow at run time, or code running
 * where CUDA API calls such as cudaMalloc are not allowed.  The kernels run on
 * a 32 MiB scratch array that is part of the library itself; every GPU that
 * loads the library holds it until the process exits.  Arguments and results
 * are those of gdr_chunk_prefill (no fusion).  The call allocates nothing.
 *  - The scratch holds a window of at least one chunk for every sequence:
 *    gdr_chunk_prefill_workspace_size(n_seqs, hv, 1, hT != NULL) must not
 *    exceed gdr_chunk_prefill_noalloc_scratch_bytes(), otherwise the call
 *    returns GDR_ERR_WORKSPACE and launches nothing (for 48 value heads:
 *    up to 8 sequences with hT given).  Longer sequences are processed in
 *    more windows, i.e. more kernel launches.
 *  - Every call made outside stream capture looks up the scratch's device
 *    address with cudaGetSymbolAddress on the current device (a device reset
 *    or a new primary context can move it).  A call made while `stream` is
 *    being captured cannot do the lookup and uses the address found by the
 *    last call outside capture on that device: make one call on the device
 *    before capturing, and none across a device reset during capture.  A
 *    first call made during capture returns GDR_ERR_UNSUPPORTED.
 *  - All calls share the one scratch array, which keeps whatever the last
 *    call left in it (no call relies on its contents: every part is written
 *    before it is read).  Calls whose work overlaps on the GPU -- on two
 *    streams, or from two threads -- race on the scratch and corrupt each
 *    other's results: serialise them.
 */
GDR_API int gdr_chunk_prefill_noalloc(const void *q, const void *k, const void *v,
                                      int64_t qk_token_stride, int64_t v_token_stride,
                                      const void *a, const void *b, const float *A_log,
                                      const float *dt_bias, float scale, int hk, int hv,
                                      const int32_t *cu_seqlens_dev,
                                      const int32_t *cu_seqlens_host, int n_seqs,
                                      const float *h0, float *hT, void *o, void *stream);

/* Size in bytes of the scratch array gdr_chunk_prefill_noalloc runs on. */
GDR_API size_t gdr_chunk_prefill_noalloc_scratch_bytes(void);

/*
 * gdr_decode_step -- one token for each of `batch` independent sequences
 * ("33B 只做 18 层 ...", §1.2: the single-step recurrent call taken when one
 * new token resumes from the cached state; "33B 只做 18 层 ..." (mhpq.cn)
 * §2.1: the single-step form of the causal conv).
 * Per sequence: conv step y = SiLU(w0 s0 + w1 s1 + w2 s2 + w3 x) over all
 * channels (rounded to bf16), the conv state rolls to (s1, s2, x); then the
 * L2 norm of q and k, the gates, and one step of the recurrence on the state,
 * which is read once and written once in place.
 *   x:          bf16 [batch][hk*128*2 + hv*128] this step's conv input [q | k | v]
 *   conv_w:     bf16 [channels][4]
 *   conv_state: bf16 [batch][3][channels], in/out (updated in place)
 *   a, b:       bf16 [batch][hv]
 *   A_log, dt_bias: fp32 [hv]
 *   state:      fp32 [batch][hv][128][128], in/out (updated in place)
 *   o:          bf16 [batch][hv][128]
 * If the bounded wait for a (sequence, value head)'s state tile runs out (the
 * device error word then reads GDR_ERR_TIMEOUT), that head writes neither its
 * state, its o row nor its v channels of the conv state; the q and k channels
 * of its key head roll only if the key head's first value head completed.
 * Treat the results of such a step as invalid.
 */
GDR_API int gdr_decode_step(const void *x, const void *conv_w, void *conv_state, const void *a, const void *b,
                    const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                    float *state, void *o, int batch, void *stream);

/*
 * gdr_decode_step_slots -- gdr_decode_step on a pool of cached states
 * ("33B 只做 18 层 ...", §1.2: the layer keeps each request's recurrent state
 * and conv state in a per-layer cache and resumes from it for the next token).
 * Row i of the batch reads and writes pool entry slot[i] of both pools; x, a,
 * b and o stay indexed by the row.  The arithmetic is that of gdr_decode_step,
 * so a row gives the bits that gdr_decode_step gives on the same inputs.
 *   conv_state_pool: bf16 [n_slots][3][channels], in/out
 *   state_pool:      fp32 [n_slots][hv][128][128], in/out
 *   slot:            int32 [batch], DEVICE memory, 4-byte aligned; read by the
 *                    kernel, so it may be written by earlier work on the stream
 *   other arguments as gdr_decode_step.
 * A slot outside [0, n_slots) (e.g. -1) marks a padding row: neither pool is
 * read or written for it and its o row is set to zero.  n_slots == 0 (both
 * pools may then be NULL) makes every row a padding row.  Two rows naming the
 * same slot in one call race: their results are undefined (every access stays
 * inside the pools).  Returns GDR_ERR_NULL for a NULL slot array or a NULL
 * pool with n_slots > 0, GDR_ERR_SHAPE for a negative batch or n_slots.
 */
GDR_API int gdr_decode_step_slots(const void *x, const void *conv_w, void *conv_state_pool, const void *a,
                                  const void *b, const float *A_log, const float *dt_bias, float scale,
                                  int hk, int hv, float *state_pool, int n_slots, const int32_t *slot,
                                  void *o, int batch, void *stream);

/*
 * gdr_chunk_prefill_slots -- gdr_chunk_prefill on a pool of cached states
 * ("33B 只做 18 层 ...", §1.2: each request's recurrent state lives in a
 * per-layer cache; a prompt fills it and later calls resume from it).
 * Sequence n reads its initial state from, and writes its final state to,
 * entry slot[n] of state_pool, in place.  With the decode's pool form this
 * serves mixed batches: new requests are prefilled into their entries and
 * running ones decode from theirs, all on one pool.
 *   q, k, v, strides, a, b, A_log, dt_bias, scale, hk, hv, cu_seqlens, o:
 *                 as gdr_chunk_prefill (no fusion)
 *   state_pool:   fp32 [n_slots][hv][128][128], in/out
 *   slot:         int32 [n_seqs], DEVICE memory, 4-byte aligned; read by the
 *                 kernels, so it may be written by earlier work on the stream
 *   init_from_pool: 1 = a sequence starts from its entry's state (a prompt
 *                 continued in a later call), 0 = from zero (a new request);
 *                 the entry is overwritten with the final state either way
 *   workspace:    at least gdr_chunk_prefill_workspace_size(n_seqs, hv, 1, 0)
 *                 bytes (the form without a final state: sequences without an
 *                 entry carry their state through the workspace)
 * A slot outside [0, n_slots) (e.g. -1) marks a sequence without an entry: it
 * starts from zero, its o rows are written, and its final state is dropped.
 * An empty sequence with an entry leaves it as it was (init_from_pool = 1) or
 * sets it to zero (0).  The arithmetic is gdr_chunk_prefill's, so o and the
 * final states equal that call's on the same initial states bit for bit.  Two
 * sequences naming the same entry in one call race (every access stays inside
 * the pool).  Returns GDR_ERR_NULL for a NULL slot array, a NULL pool with
 * n_slots > 0 or a NULL input with tokens to process, GDR_ERR_SHAPE for a
 * negative n_slots or init_from_pool not 0 or 1, GDR_ERR_WORKSPACE for a
 * workspace below the size above.
 */
GDR_API int gdr_chunk_prefill_slots(const void *q, const void *k, const void *v, int64_t qk_token_stride,
                                    int64_t v_token_stride, const void *a, const void *b, const float *A_log,
                                    const float *dt_bias, float scale, int hk, int hv,
                                    const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seqs,
                                    float *state_pool, int n_slots, const int32_t *slot, int init_from_pool,
                                    void *o, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr_linear -- a projection of the layer: y = x W^T in bf16 with fp32
 * accumulation, on the tensor cores ("33B 只做 18 层 ...", §2 parameter table:
 * the hidden state of 5120 is projected to q|k|v (10 240), z (6144), a and b
 * (48 each), and the gated norm's output (6144) back to 5120).
 *   x: bf16 [M][K] row-major (rows of the activations, e.g. tokens x hidden)
 *   w: bf16 [N][K] row-major (the weight as stored for out = in W^T)
 *   y: bf16 [M][N] row-major, written; must not overlap x or w (GDR_ERR_ALIAS)
 * y[m][n] = round_bf16(sum_k x[m][k] w[n][k]), the sum in fp32.  N and K must
 * be multiples of 8 (rows of whole 16-byte chunks) and M, N, K positive with
 * N <= 2^24 (GDR_ERR_SHAPE); M == 0 is a no-op.  Pointers 16-byte aligned
 * (GDR_ERR_ALIGN).  Asynchronous on `stream`; a bounded wait that runs out
 * sets GDR_ERR_TIMEOUT in the device error word and leaves y incomplete.
 */
GDR_API int gdr_linear(const void *x, const void *w, void *y, int64_t M, int64_t N, int64_t K, void *stream);

/*
 * gdr_gated_rmsnorm -- gated RMSNorm over rows of d values
 * ("Agnes-3.0-Flash 深度解析", 注意力层的细节: gated RMS-norm; the z
 * projection of width 6144 = 48 x 128 in the parameter table of
 * "33B 只做 18 层 ...", §2):
 *     y = o / sqrt(mean(o^2) + eps) * w * SiLU(z)    (fp32 math, bf16 out)
 *   o, z, y: bf16 [rows][d], d == 128;  w: fp32 [d] or NULL (ones).
 *   y may equal o (in place).
 */
GDR_API int gdr_gated_rmsnorm(const void *o, const void *z, const float *w, float eps, int64_t rows, int d,
                      void *y, void *stream);

/*
 * Text of the last host-side failure of a call made from this thread: which
 * step failed and the CUDA error string (empty when the last call succeeded).
 * The pointer stays valid until the next call from the same thread.
 */
GDR_API const char *gdr_last_error_string(void);

/*
 * Read and clear the device-side error word (0 = none, else a gdr_status_t
 * such as GDR_ERR_TIMEOUT) after the work queued on `stream` completes.
 * This call synchronises `stream`.
 */
GDR_API int gdr_get_device_error(int *error_out, void *stream);

/*
 * gdr_debug_wait_timeout -- self-test of the kernels' bounded waits (no
 * counterpart in the pages: a diagnostic of this library).
 * Launches one CTA that allocates tensor memory and then waits, with the
 * wait helpers the kernels use, on an mbarrier that nothing arrives at:
 *   kind 0: the poll-count bound of the prep, conv and decode kernels;
 *   kind 1: the clock bound of the prefill's state chain (all warps wait).
 * `limit` is the bound (polls for kind 0, SM clock cycles for kind 1; at most
 * 2^31).  When it runs out the kernel records GDR_ERR_TIMEOUT in the device
 * error word, releases its tensor memory and returns; it writes 0 to
 * result_dev[0] (1 would mean the wait completed).  No copy or MMA is in
 * flight while it waits.  Returns GDR_ERR_SHAPE for another kind or a limit
 * of 0 or above 2^31, GDR_ERR_NULL without result_dev.
 */
GDR_API int gdr_debug_wait_timeout(int kind, unsigned long long limit, int *result_dev, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
