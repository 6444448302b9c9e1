/*
 * pv.h - same-step KV chunk attention for B200 (sm_100a), C ABI.
 *
 * The operation (PhysisServe Wan2.2-5B model card, "Inference profile" and
 * the paragraph below it): video is generated chunk by chunk in latent space.
 * The first chunk holds 3 latent frames, every later chunk 1 frame, and each
 * chunk is denoised in 4 steps.  At denoising step s a chunk attends to the
 * K/V that earlier chunks recorded at the same step s, plus a sink: the clean
 * K/V of the first chunk, recorded by one extra pass at sigma = 0.  The
 * history holds at most R recent chunks besides the sink.  Around the
 * attention sit the 3D (frame, height, width) RoPE of q and k (blog
 * "Learning Video Generation from the Wan2.2 Source Code", chapter 4, "3D
 * RoPE") and the flow-matching Euler update x += (sigma_next - sigma) * v
 * (same blog, chapter 5, "UniPC", and chapter 1).
 *
 * Conventions for every entry point
 *  - Ownership: the caller allocates every device buffer and owns the CUDA
 *    stream.  The library never allocates device memory; a pv_kv handle keeps
 *    host bookkeeping and the caller's pointers only.
 *  - Streams: `cuda_stream` is a cudaStream_t passed as void* (NULL = the
 *    legacy default stream).  Every kernel call is asynchronous on it.
 *  - Errors: every call returns a pv_status.  Arguments and shapes are
 *    checked on the host before any launch; nothing aborts across the ABI.
 *    A fault of an earlier asynchronous launch surfaces as PV_ERR_CUDA on a
 *    later call.  pv_last_error() gives a one-line message for the calling
 *    thread's most recent failure.
 *  - Workspaces hold a launch's scratch state: split-KV partial results and
 *    arrival counters for attention (a handle's workspace for pv_chunk_attn,
 *    the `ws` argument for pv_attn_dense and pv_attn_varlen), the projected
 *    q/k/v and their sums of squares for pv_qkv_rope_append.  Launches that
 *    use one workspace must not overlap on the GPU: issue them on one CUDA
 *    stream, or order them with events.  The host side of a handle is
 *    guarded by a mutex.
 *  - Element types: "bf16" is IEEE bfloat16 (2 bytes), "f32" is float.
 *  - Device pointers must be 16-byte aligned; the KV store must be 256-byte
 *    aligned.
 *  - Notation: T = frame_w * frame_h tokens per latent frame, F0 =
 *    first_frames, R = ring_slots, H = heads, D = head_dim, Ltot = (F0 + R)*T
 *    key rows per (layer, step, stream, head).
 */
#ifndef PV_H
#define PV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PV_API __attribute__((visibility("default")))
#else
#define PV_API
#endif

typedef int pv_status;
#define PV_OK                   0
#define PV_ERR_INVALID_ARG      1  /* null pointer, bad enum, misaligned pointer */
#define PV_ERR_SHAPE            2  /* sizes that the kernels do not support */
#define PV_ERR_CAPACITY         3  /* a buffer smaller than required */
#define PV_ERR_STATE            4  /* a call out of order in the chunk schedule */
#define PV_ERR_UNSUPPORTED_ARCH 5  /* the current device is not sm_100 */
#define PV_ERR_CUDA             6  /* a CUDA runtime or driver error */
#define PV_ERR_TIMEOUT          7  /* a device-side wait gave up (see pv_kv_poll_device_error) */

/* Step index of the sigma = 0 bootstrap pass that records the sink. */
#define PV_STEP_SINK (-1)

/* Largest ring (slots) and stream count that one handle supports. */
#define PV_MAX_RING    64
#define PV_MAX_STREAMS 64

/* Phases of one stream (model card, "Inference profile"). */
#define PV_PHASE_NEW    0  /* no chunk yet */
#define PV_PHASE_FIRST  1  /* the first chunk (F0 frames) is being denoised */
#define PV_PHASE_BOOT   2  /* the sigma = 0 pass over the clean first chunk */
#define PV_PHASE_STEADY 3  /* chunks of one frame, reading sink + ring */

/* Geometry and capacity of a KV store. */
typedef struct pv_kv_config {
    int layers;        /* transformer layers that keep a history (30 for Wan2.2-5B) */
    int heads;         /* H */
    int head_dim;      /* D: 64 or 128 */
    int frame_w;       /* tokens per row of a latent frame (40 at 1280 px) */
    int frame_h;       /* token rows of a latent frame (22 at 704 px);
                          frame_w * frame_h <= 2^24 */
    int first_frames;  /* F0: latent frames of the first chunk (3) */
    int ring_slots;    /* R: recent chunks kept besides the sink (18), 1..PV_MAX_RING */
    int steps;         /* denoising steps per chunk (4) */
    int max_streams;   /* independent generation streams sharing the store */
    int rope_pairs_t;  /* RoPE pairs of the time axis   (22 for D = 128, 12 for D = 64) */
    int rope_pairs_h;  /* RoPE pairs of the height axis (21 for D = 128, 10 for D = 64) */
    int rope_pairs_w;  /* RoPE pairs of the width axis  (21 for D = 128, 10 for D = 64) */
    int max_frames;    /* largest latent-frame index + 1 that RoPE may see, <= 2^20 */
    double rope_theta; /* RoPE base (10000) */
} pv_kv_config;

/* Host bookkeeping of one stream.  pv_kv_get_state fills it; pv_kv_set_state
 * restores it (checkpoint / resume of the schedule position). */
typedef struct pv_kv_state {
    int phase;      /* PV_PHASE_* */
    int chunk;      /* current chunk index j (0 = the first chunk, -1 before it) */
    int fill;       /* ring slots holding a chunk: min(j, R) for j >= 1 */
    int slot;       /* ring slot of the current chunk: (j - 1) mod R, or -1 */
    int frame0;     /* latent-frame index of the current chunk's first frame */
    int nframes;    /* latent frames in the current chunk */
    int n_queries;  /* tokens of the current chunk: nframes * T */
    int n_keys;     /* keys the current chunk reads at one step */
    int slot_frame[PV_MAX_RING]; /* latent frame held by each slot, -1 if empty */
} pv_kv_state;

typedef struct pv_kv_s* pv_kv;

/* Library version string (static storage). */
PV_API const char* pv_version(void);

/* Copies the calling thread's last error message into buf (always
 * NUL-terminated when len > 0).  Returns the status of that failure. */
PV_API pv_status pv_last_error(char* buf, size_t len);

/* Sizes of the two caller-allocated device buffers for cfg.
 *  kv_bytes: the KV store, 2 * layers * steps * max_streams * H * Ltot * D
 *            bf16 (K region followed by V region).
 *  ws_bytes: the workspace: RoPE cos/sin table, split-KV partial results,
 *            arrival counters, the fused projection's flags and a device
 *            error word. */
PV_API pv_status pv_kv_required_bytes(const pv_kv_config* cfg, size_t* kv_bytes, size_t* ws_bytes);

/* Creates a handle over caller buffers.  Checks cfg (D in {64,128}, RoPE
 * pairs summing to D/2, 1 <= R <= PV_MAX_RING, ...), checks that the current
 * device is sm_100, builds the RoPE table on the host in fp64, uploads it
 * (synchronous cudaMemcpy) and zero-fills the store and the workspace
 * (synchronous cudaMemset), so that unused key rows hold zeros.  All streams
 * start in PV_PHASE_NEW.
 * Passing kv_dev == NULL and ws_dev == NULL makes a bookkeeping-only handle:
 * no device is touched, the schedule calls work, kernel calls return
 * PV_ERR_STATE.  The handle is freed by pv_kv_destroy. */
PV_API pv_status pv_kv_init(pv_kv* out, const pv_kv_config* cfg, void* kv_dev, size_t kv_bytes,
                     void* ws_dev, size_t ws_bytes);
PV_API pv_status pv_kv_destroy(pv_kv kv);

/* Starts the next chunk of `stream` (model card, "Inference profile": the
 * first chunk has F0 frames, every later one 1 frame).  NEW -> FIRST needs
 * nframes == F0; BOOT or STEADY -> STEADY needs nframes == 1 and advances j,
 * taking ring slot (j - 1) mod R.  Any other use returns PV_ERR_STATE and
 * leaves the state unchanged. */
PV_API pv_status pv_kv_begin_chunk(pv_kv kv, int stream, int nframes);

/* Starts the sigma = 0 bootstrap pass of `stream` over its clean first chunk
 * (model card: "receives an additional forward pass to build the persistent
 * sink").  FIRST -> BOOT; any other phase returns PV_ERR_STATE. */
PV_API pv_status pv_kv_begin_sink(pv_kv kv, int stream);

PV_API pv_status pv_kv_get_state(pv_kv kv, int stream, pv_kv_state* out);
/* Restores a state taken by pv_kv_get_state (fields are re-validated and the
 * derived ones recomputed).  The store contents are the caller's to restore. */
PV_API pv_status pv_kv_set_state(pv_kv kv, int stream, const pv_kv_state* st);

/* Element offsets (in bf16 units from kv_dev) of key row `key` of
 * (layer, step, stream, head) in the K and the V region.  step is 0..steps-1.
 * Rows 0..F0*T-1 are the sink, row F0*T + slot*T + t is token t of a slot. */
PV_API pv_status pv_kv_row_offset(pv_kv kv, int layer, int step, int stream, int head, int key,
                           size_t* k_elem, size_t* v_elem);

/* 3D RoPE of q and k plus the append of (k_rot, v) into the per-step store,
 * for each listed stream at its current chunk.
 *  streams[n_streams]: distinct stream ids (host array).
 *  step: 0..steps-1, or PV_STEP_SINK for the bootstrap pass.
 *    FIRST phase, step s: k_rot, v go to the sink rows of step buffer s.
 *    PV_STEP_SINK (phase BOOT, see pv_kv_begin_sink): k_rot, v go to the
 *      sink rows of every step buffer.
 *    STEADY phase, step s: k_rot, v go to ring slot (j - 1) mod R of step s.
 *  q, k, v: bf16 [sum_i Lq_i][H][D], the streams' tokens packed in list
 *    order, Lq_i = nframes_i * T, tokens of a frame row-major (h * frame_w + w).
 *  q_rot: bf16 output, head-major per stream: stream i's block starts at row
 *    H * (sum_{i'<i} Lq_i') and is [H][Lq_i][D].
 *  Token t of the chunk sits at latent frame frame0 + t / T, height
 *  (t % T) / frame_w, width t % frame_w; pair p of a head rotates by
 *  pos_axis(p) * theta^(-2 k / (2 * pairs_axis)), k = p's index in its axis
 *  block, as the complex product (x[2p] + i x[2p+1]) e^{i angle}; fp32
 *  arithmetic on a table built in fp64, rounded once to bf16. */
PV_API pv_status pv_rope_append(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                         const void* q, const void* k, const void* v, void* q_rot,
                         void* cuda_stream);

/* Workspace bytes of pv_qkv_rope_append for `tokens` tokens (all listed
 * streams together) of width dim = heads * head_dim. */
PV_API pv_status pv_qkv_ws_bytes(int tokens, int dim, size_t* ws_bytes);

/* The q, k, v projection with QK-Norm, then what pv_rope_append does
 * (blog chapter 4, end of "3D RoPE": q and k each pass through their linear
 * layer and an RMSNorm; v through its linear layer):
 *   y = x w^T + bias                       (f32 accumulate)
 *   q = RMSNorm(y[:, 0:dim]) * g_q,  k = RMSNorm(y[:, dim:2 dim]) * g_k,
 *   v = y[:, 2 dim:3 dim],  RMSNorm(u) = u / sqrt(mean(u^2) + eps),
 * over the whole vector of a token (all heads), heads split afterwards
 * (feature f to head f / head_dim); then 3D RoPE of q and k and the append
 * of k, v into the per-step store exactly as pv_rope_append, q_rot likewise.
 *  x: bf16 [tokens][dim] (the listed streams' tokens back to back, in list
 *     order), w: bf16 [3 dim][dim] (W_q, W_k, W_v rows, a linear layer's
 *     [out][in]), bias: f32 [3 dim], g_q, g_k: f32 [dim] (all 16-byte
 *     aligned), eps > 0.  Misaligned pointers: PV_ERR_INVALID_ARG.
 *  ws: device workspace of pv_qkv_ws_bytes, 256-byte aligned (holds y in
 *     f32 and the per-token sums of squares; no need to clear it).
 * When every tile of the GEMM can be resident at once (tokens <= 1024 at
 * dim 3072: the steady chunk) and the RoPE table fits in shared memory
 * beside a tile, one cooperative launch: a tcgen05 GEMM whose epilogue adds
 * the bias, writes each token's sum of squares over its tile, raises its
 * flag in the handle's workspace, waits (bounded, about a second; a wait
 * that gives up sets the handle's device error word) until every tile of
 * the token's q or k has done so, adds their sums in tile order, then
 * applies the norm, the gain and the rotation to the accumulator and writes
 * bf16 q_rot and the K/V rows; y is not written.  Otherwise a memset and
 * two launches: the GEMM writes y and adds the sums of squares, and the
 * RoPE / append kernel applies the norm as it reads y.  Both round each
 * output once to bf16.  The handle's workspace is used either way: calls
 * on one handle must not overlap on the GPU. */
PV_API pv_status pv_qkv_rope_append(pv_kv kv, int n_streams, const int* streams, int layer,
                                    int step, const void* x, const void* w, const float* bias,
                                    const float* g_q, const float* g_k, float eps, void* q_rot,
                                    void* ws, size_t ws_bytes, void* cuda_stream);

/* Chunk attention of each listed stream at its current chunk, one launch:
 *  o[q] = sum_k softmax_k(q_rot . k_rot / sqrt(D)) v_k over the stream's key
 *  set at (layer, step): FIRST -> its own F0*T keys of step s; PV_STEP_SINK
 *  (phase BOOT) -> its own clean keys; STEADY -> sink + the `fill` ring slots
 *  of step s (F0*T + fill*T keys).  No causal mask.
 *  q_rot: as written by pv_rope_append with the same stream list.
 *  out: bf16 [sum_i Lq_i][H][D], token-major like q.
 *  lse: optional f32 [sum_i Lq_i][H], natural-log log-sum-exp of the logits.
 *  Computes in bf16 on the tensor cores with f32 accumulation and softmax. */
PV_API pv_status pv_chunk_attn(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                        const void* q_rot, void* out, float* lse, void* cuda_stream);

/* 3D RoPE over a whole clip of n_tokens = nframes * T tokens starting at
 * latent frame frame0, with the handle's geometry and table (for full
 * bidirectional attention over a video):
 *  q, k, v: bf16 [n_tokens][H][D]; q_rot, k_rot, v_hm: bf16 [H][n_tokens][D]
 *  (v_hm is v moved to head-major, unrotated). */
PV_API pv_status pv_rope_dense(pv_kv kv, int n_tokens, int frame0, const void* q, const void* k,
                        const void* v, void* q_rot, void* k_rot, void* v_hm, void* cuda_stream);

/* Workspace bytes that pv_attn_dense needs for (Lq, Lk, H, D). */
PV_API pv_status pv_attn_dense_ws_bytes(int n_q, int n_k, int heads, int head_dim, size_t* ws_bytes);

/* Plain softmax attention on explicit head-major buffers, the same kernel as
 * pv_chunk_attn:  q [H][n_q][D], k and v [H][n_k][D] bf16, out [n_q][H][D]
 * bf16, lse optional f32 [n_q][H].  1 <= n_q, n_k <= 2^30 and H * n_q,
 * H * n_k < 2^31 (rows of one tensor map), else PV_ERR_SHAPE.  Key rows
 * past n_k inside a 128-key tile are read from the next head (or as zeros
 * past the buffer) and masked out, so k and v must hold finite values.
 * ws: device workspace of pv_attn_dense_ws_bytes bytes, zero-filled by the
 * caller before its first use (the kernels leave it zeroed again).  Its first
 * int is the device error word: nonzero after a call whose bounded device
 * wait gave up (that call's out / lse are then incomplete).
 * pv_attn_poll_device_error reads it and, if set, zeroes the workspace
 * again. */
PV_API pv_status pv_attn_dense(const void* q, const void* k, const void* v, int n_q, int n_k,
                        int heads, int head_dim, void* out, float* lse, void* ws,
                        size_t ws_bytes, void* cuda_stream);

/* Workspace bytes that pv_attn_varlen needs for these sequence lengths. */
PV_API pv_status pv_attn_varlen_ws_bytes(int n_seqs, const int* n_q, const int* n_k, int heads,
                                         int head_dim, size_t* ws_bytes);

/* Softmax attention of n_seqs independent sequences of ragged lengths in one
 * launch, the same kernel as pv_attn_dense.  Its use here is the DiT's
 * cross-attention (blog chapter 3, "Where Did the Prompt Go?": each layer's
 * video tokens query the prompt's text context, up to 512 vectors, trimmed
 * to the prompt's real length; chapter 4: the context holds no sequence
 * positions, so no RoPE, and no mask), one sequence per prompt.
 *  n_q, n_k: HOST arrays of n_seqs lengths (1 <= n_seqs <= PV_MAX_STREAMS);
 *    n_q[i] = 0 skips sequence i; n_q[i] > 0 needs n_k[i] >= 1; every length
 *    <= 2^30 and H * sum n_q, H * sum n_k < 2^31, else PV_ERR_SHAPE.
 *  q: the sequences' head-major blocks back to back, bf16: block i is
 *    [H][n_q[i]][D] and starts at row H * (n_q[0] + ... + n_q[i-1]).
 *  k, v: likewise [H][n_k[i]][D] blocks.  Rows past a block's last key inside
 *    a 128-key tile are read from the next block (or as zeros past the
 *    buffer) and masked out, so k and v must hold finite values.
 *  out: bf16 [sum n_q][H][D], token-major, sequence i from token
 *    n_q[0] + ... + n_q[i-1].  lse: optional f32 [sum n_q][H].
 *  ws: device workspace of pv_attn_varlen_ws_bytes bytes, zero-filled before
 *    its first use, 256-byte aligned.  Its first int is the device error
 *    word, as for pv_attn_dense (pv_attn_poll_device_error). */
PV_API pv_status pv_attn_varlen(const void* q, const void* k, const void* v, int n_seqs,
                                const int* n_q, const int* n_k, int heads, int head_dim,
                                void* out, float* lse, void* ws, size_t ws_bytes,
                                void* cuda_stream);

/* The work plan that pv_attn_varlen would launch for these lengths on a GPU
 * with n_sm SMs and a workspace of partial_slots split-KV slots (head_dim
 * 128), without launching anything: host only.  Items are (sequence, head,
 * 256-query block), each a run of ceil(n_k / 128) key tiles, laid out
 * query-block-major and end to end.
 *  grid: CTAs; ranges: host array of at least min(n_sm, 160) + 1 entries.
 *  mode 0, stream-K: CTA c processes the key tiles [ranges[c],
 *    ranges[c + 1]) of the list (equal shares; an item split between CTAs is
 *    merged by the last of them to arrive).
 *  mode 1, whole items at run time: the sequences are put in decreasing
 *    order of key tiles and each CTA takes the next whole item from a
 *    counter until none is left (longest first); nothing is split.
 *    ranges[0] = 0, ranges[grid] = the total key tiles, the others -1. */
PV_API pv_status pv_attn_plan(int n_seqs, const int* n_q, const int* n_k, int heads, int n_sm,
                              int partial_slots, int* grid, int* mode, long long* ranges);

/* Dense attention like pv_attn_dense (same layouts, same kernel), for
 * callers that cannot allocate device memory where they call it: code inside
 * a custom allocator or memory-pool callback, plugins whose host framework
 * owns all device allocations, latency-critical paths that must not touch
 * the allocator.  It takes no workspace and calls no allocating routine:
 * its split-KV scratch is a fixed 8 MiB array inside the library, held by
 * every GPU that loads the library until the process exits.  The pages
 * describe no counterpart of this call; it is a property of this library.
 *  - Limit: heads * ceil(n_q / 256) * 2 <= 16384 query tiles, else
 *    PV_ERR_CAPACITY with a message naming the limit (use pv_attn_dense).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - Every call shares the one array and clears the part it needs on
 *    cuda_stream; calls whose executions overlap on the GPU (other streams,
 *    other host threads) race on it and must be serialised by the caller.
 *  - A bounded device wait that gives up (about one second) leaves out / lse
 *    incomplete and sets the array's device error word, which the next call
 *    clears: read it after the call with pv_attn_poll_device_error(NULL, 0,
 *    ...) on the same stream. */
PV_API pv_status pv_attn_dense_noalloc(const void* q, const void* k, const void* v, int n_q,
                                       int n_k, int heads, int head_dim, void* out, float* lse,
                                       void* cuda_stream);

/* Flow-matching Euler update in place (blog chapter 5, "UniPC"):
 *  x[i] += dsigma * v[i] for i < n, f32, one fused multiply-add per element.
 *  dsigma = sigma_next - sigma (negative while denoising), computed by the
 *  caller in fp64 and passed rounded to f32. */
PV_API pv_status pv_euler_step(float* x, const float* v, size_t n, float dsigma, void* cuda_stream);

/* Shifted sigma schedule of n_steps denoising steps (blog chapter 5, "shift:
 * Where the 40 Stops Land"): a uniform grid u_i = sigma_max * (1 - i/n_steps),
 * i < n_steps, mapped by sigma = shift * u / (1 + (shift - 1) * u), then a
 * final 0.  sigmas_out: host array of n_steps + 1 doubles.  timesteps_out
 * (optional, n_steps ints): floor(1000 * sigma_i), the 1000-tick scale of
 * the blog's chapter 1.  sigma_max <= 0 selects 1 - 1/1000, which with shift
 * 12 and 40 steps gives the blog's printed 999, 997, 995, 993, 990, 988.
 * Host only, fp64. */
PV_API pv_status pv_sigma_schedule(int n_steps, double shift, double sigma_max,
                                   double* sigmas_out, int* timesteps_out);

/* Euler update on the classifier-free-guided velocity, in place (blog
 * chapter 5, "CFG"): x[i] += dsigma * (v_uncond[i] + guide_scale *
 * (v_cond[i] - v_uncond[i])), f32; the guided velocity is never stored. */
PV_API pv_status pv_euler_cfg_step(float* x, const float* v_cond, const float* v_uncond,
                                   size_t n, float guide_scale, float dsigma,
                                   void* cuda_stream);

/* Clean-data estimate of flow matching (blog chapter 1): x0[i] = x[i] -
 * sigma * v[i], f32, one fused multiply-add per element; x0 may alias x. */
PV_API pv_status pv_x0_estimate(float* x0, const float* x, const float* v, size_t n,
                                float sigma, void* cuda_stream);

/* Reads (synchronously) and clears the device error word that the kernels of
 * this handle set when a bounded device-side wait gives up.  *code is 0 when
 * no wait timed out; otherwise the call returns PV_ERR_TIMEOUT and also
 * re-zeroes the workspace's counters (split-merge arrivals, run-time item
 * hand-out), which an aborted launch may have left part counted. */
PV_API pv_status pv_kv_poll_device_error(pv_kv kv, int* code);

/* Reads and clears the device error word of an attention workspace: ws and
 * ws_bytes as given to pv_attn_dense or pv_attn_varlen, or ws = NULL for the
 * fixed scratch of pv_attn_dense_noalloc (ws_bytes ignored).  Waits for
 * cuda_stream first (synchronous).  *code is 0 when no device wait gave up;
 * otherwise the call zeroes the workspace (the scratch's error word only,
 * since each no-alloc call clears its counters itself) and returns
 * PV_ERR_TIMEOUT: the output of the call that timed out is incomplete.
 * A ws that is not 256-byte aligned or under 256 bytes: PV_ERR_INVALID_ARG. */
PV_API pv_status pv_attn_poll_device_error(void* ws, size_t ws_bytes, int* code,
                                           void* cuda_stream);

/* Failure-path self-test of the workspace entry points: one device-side wait
 * on a barrier that nothing arrives on gives up after about one second and
 * records a timeout in the error word of ws (NULL: the no-alloc scratch),
 * exactly as a wait of the attention kernel would; the context stays usable.
 * Asynchronous on cuda_stream. */
PV_API pv_status pv_attn_selftest_wait_timeout(void* ws, void* cuda_stream);

/* Failure-path self-test: launches one device-side wait on a barrier that
 * nothing ever arrives on.  Like every wait of the attention kernel it gives
 * up after about one second, records a timeout in this handle's device error
 * word and returns, leaving the GPU context usable; pv_kv_poll_device_error
 * then reports PV_ERR_TIMEOUT.  Asynchronous on cuda_stream. */
PV_API pv_status pv_kv_selftest_wait_timeout(pv_kv kv, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* PV_H */
