/*
 * gdn.h - C ABI of the frame-wise Gated DeltaNet (GDN) frame-scan library for NVIDIA B200
 * (sm_100a). Every entry point is asynchronous on the caller's CUDA stream.
 *
 * The layer (one head; sources: "NVIDIA SANA-WM: минутное 720p видео с одной видеокарты",
 * gen-hub.ru, section "Архитектура: четыре нетривиальных решения" -- decay gate gamma,
 * delta-rule residual correction beta, constant D x D state, key scale 1/sqrt(D*S); "SANA-WM:
 * Efficient Minute-Scale World Modeling with Hybrid Linear Diffusion Transformer", chatpaper.ai
 * abstract, design (1) -- the GDN is frame-wise):
 *
 *     k' = key_scale * k
 *     A_t = K'_t^T K'_t,   B_t = V_t^T K'_t                       (D x D each)
 *     S_t = gamma_t * S_{t-1} (I - beta_t A_t) + beta_t B_t        (fp32 state, row v, col k)
 *     O_t = Q_t S_t^T                                              (bf16 output)
 *
 * so attention is bidirectional within a frame (every token of frame t reads S_t) and causal
 * across frames.
 *
 * Common conventions
 *  - Pointers are DEVICE pointers owned by the caller; the library never frees them.
 *  - q, k, v, out: [B, T, N, H, D] bfloat16 (gdn_bf16 = raw bf16 bits), contiguous, token-major
 *    (frame t of head h is N rows of D values with a row stride of H*D elements).
 *  - gamma, beta: [B, T, H] float32 (decay gate and delta-rule strength, used as given).
 *  - state: [B, H, D, D] float32, row-major, row = value index, column = key index, so that
 *    S k is a value. A NULL state_in means S_0 = 0; a NULL state_out skips the final store.
 *  - D must be a multiple of 8 in [8, 128]; B, H, T, N >= 1; every tensor pointer must be
 *    16-byte aligned (GDN_ERR_MISALIGNED otherwise).
 *  - key_scale (every GDN entry point that takes one): 0 selects the pages' key scale
 *    1/sqrt(D*N), computed by the library in double precision and rounded to f32 (D the head dim,
 *    N the tokens per frame of the call; gen-hub.ru article, "Архитектура"); any other value
 *    must be finite and > 0 and is used as given (1 for unscaled keys). Negative, NaN or
 *    infinite values return GDN_ERR_INVALID_ARG.
 *  - out must not overlap q, k or v (GDN_ERR_INVALID_ARG). state_out may equal state_in
 *    (in-place streaming); any other partial overlap is undefined.
 *  - Errors found on the host are returned before anything is launched. Launch failures return
 *    GDN_ERR_CUDA. Kernels never trap: a device-side wait that exceeds its time limit records
 *    GDN_ERR_TIMEOUT in a per-device status word that gdn_sync_status() reports.
 *  - The library keeps one cached device workspace per GPU (see gdn_workspace_bytes); it grows
 *    on demand in stream order (cudaFreeAsync of the old buffer and cudaMallocAsync of the new
 *    one on the caller's stream, from the device's default memory pool: no device-wide
 *    synchronisation; refused with GDN_ERR_NO_MEMORY while the stream is being captured) and is
 *    shared by all calls on that GPU: calls on different streams of the same GPU must not run
 *    concurrently (order them, e.g. by events). gdn_release_workspace() frees it.
 *  - GDN_POISON_WORKSPACE=1 (testing aid, read once per process): every call first fills the
 *    workspace bytes it uses with 0xFF (NaN as f32 and bf16) on its stream, so that a kernel
 *    reading workspace it has not written shows up as NaN in the results.
 *  - No CPU fallback exists: without a CUDA device every call returns GDN_ERR_CUDA.
 *
 * Environment (read once per process unless stated):
 *  - GDN_WAIT_LIMIT_MS: limit of every device-side bounded wait (default 4000).
 *  - GDN_FUSED_RING, GDN_FUSED_SRING, GDN_FUSED_STATS_PCT: ring depths of the fused forward's
 *    A_t/B_t and S_t hand-off (default 8 and 16 frames per head) and the share of the non-chain
 *    SMs given to the statistics role (default 54 %).
 *  - GDN_CHUNK_LEN: frames per chunk of the chunked forward (read on every call; 0 or unset:
 *    chosen per problem).
 *  - GDN_HOST_SEGMENT_FRAMES: frames per segment of gdn_frame_forward_host (read on every call).
 *  - GDN_BWD_SEGMENT_FRAMES: frames per segment of gdn_frame_backward's reverse state chain when
 *    its gradient passes overlap the chain (default 240; read on every call).
 *  - GDN_TEST_WITHHOLD_FRAME: test hook only. The fused forward computes but never publishes the
 *    statistics of this frame of head 0, so the call ends with GDN_ERR_TIMEOUT (after the wait
 *    limit) instead of a result; used to test failure detection without faulting the GPU.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* A cudaStream_t. NULL means the legacy default stream. */
typedef struct CUstream_st* gdn_stream_t;
/* Raw bfloat16 bits. */
typedef uint16_t gdn_bf16;

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1, /* null pointer, size out of range, overlapping out, bad scale */
  GDN_ERR_UNSUPPORTED = 2, /* head dim not supported by this entry point */
  GDN_ERR_MISALIGNED = 3,  /* a tensor pointer is not 16-byte aligned */
  GDN_ERR_NO_MEMORY = 4,   /* workspace allocation failed (or growth during capture) */
  GDN_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  GDN_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out (from gdn_sync_status) */
  GDN_ERR_SCRATCH_LIMIT = 7 /* gdn_frame_forward_noalloc: problem too large for its scratch */
} gdn_status;

/*
 * gdn_frame_forward - frame-wise GDN over a whole clip of T frames.
 * Computes out (all T frames) and, if state_out != NULL, S_T.
 * key_scale: the scale applied to keys; 0 selects the pages' 1/sqrt(D*N) (see above).
 * Workspace: gdn_workspace_bytes(B, H, T, N, D) bytes at most (three-kernel path: per-frame
 * A_t, B_t, S_t; fused path: per-head rings of A_t, B_t, S_t and hand-off flags; chunked path:
 * the three-kernel workspace plus per chunk one record of composed maps and one start state).
 */
gdn_status gdn_frame_forward(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                             const float* gamma, const float* beta, const float* state_in,
                             gdn_bf16* out, float* state_out, int B, int H, int T, int N, int D,
                             float key_scale, gdn_stream_t stream);

/*
 * gdn_frame_forward_rope - gdn_frame_forward on q and k rotated by the 3D rotary position
 * embedding of gdn_rope_3d (see there for the reading of the SANA-Video talk transcript's 3D
 * RoPE), with the rotation fused into the layer's kernels: the statistics kernel rotates each K
 * tile and the output kernel each Q tile in shared memory, between the TMA load and the tensor
 * cores, so q and k are read once and never rewritten. The result equals gdn_rope_3d of q and of
 * k (same f32 arithmetic and bf16 rounding of the rotated values) followed by gdn_frame_forward.
 * Arguments: those of gdn_frame_forward, then the latent grid of a frame (grid_h * grid_w == N,
 * token n at row n / grid_w, column n % grid_w), the rotary base (> 1, finite; 10000 is usual)
 * and t_offset (>= 0, the absolute index of the clip's first frame, so a resumed clip continues
 * its time positions). Host-side errors as gdn_frame_forward and gdn_rope_3d. Same path choice
 * (fused, three kernels, chunked) and workspace as gdn_frame_forward, plus a per-GPU cos/sin
 * table of 8 * (T * l_t + grid_h * l_h + grid_w * l_w) bytes (l_t, l_h, l_w as under
 * gdn_rope_3d; grown like the workspace, freed by gdn_release_workspace), computed by one extra
 * launch on `stream`. The kernels copy the table's grid-row and grid-column entries into shared
 * memory (256 bytes per grid row and per grid column) when grid_h + grid_w <= 127, and read them
 * from the table in global memory otherwise; either way the result is the same.
 */
gdn_status gdn_frame_forward_rope(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                  const float* gamma, const float* beta, const float* state_in,
                                  gdn_bf16* out, float* state_out, int B, int H, int T, int N,
                                  int D, float key_scale, int grid_h, int grid_w,
                                  float rope_base, int t_offset, gdn_stream_t stream);

/*
 * gdn_frame_forward_fp8 - gdn_frame_forward on 8-bit E4M3 q, k, v with one scale per
 * (batch, frame, head) (the SANA-Streaming entry of the jefxiong.cn AIGC digest, 2026-06-01,
 * item 1, contribution (3): mixed-precision quantisation to keep the tensor cores busy; the
 * pages give no quantiser, so the layer is defined on the dequantised values).
 *
 * q, k, v: [B, T, N, H, D] E4M3 codes (OCP 8-bit floating point, no infinities), device
 * pointers; q_scale, k_scale, v_scale: [B, T, H] f32, so that q[b,t,n,h,:] = decode(q8) *
 * q_scale[b,t,h] (likewise k, v). gamma, beta, state_in, out (bf16), state_out, key_scale: as
 * gdn_frame_forward. The kernels convert the codes to bf16 in shared memory (exact) and apply
 * the scales in their f32 epilogues (A gets key_scale^2 k_scale^2, B key_scale k_scale v_scale,
 * O q_scale), so the result is the bf16 layer's on the dequantised inputs up to f32 rounding
 * while q, k, v cost one byte per element to read.
 * Supported head dims: 64 < D <= 128, D % 16 == 0 (GDN_ERR_UNSUPPORTED otherwise). The same
 * path choice as gdn_frame_forward (fused, three kernels, chunked) and the same workspace.
 */
gdn_status gdn_frame_forward_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v,
                                 const float* q_scale, const float* k_scale,
                                 const float* v_scale, const float* gamma, const float* beta,
                                 const float* state_in, gdn_bf16* out, float* state_out, int B,
                                 int H, int T, int N, int D, float key_scale,
                                 gdn_stream_t stream);

/*
 * gdn_frame_forward_host - gdn_frame_forward on a clip held in HOST memory.
 * (No counterpart in the paper: a deployment variant for clips that do not stay on the GPU,
 * e.g. minute-long videos whose activations are kept in host memory between layers.)
 *
 * q, k, v, gamma, beta, out and the nullable state_in / state_out are HOST pointers with the
 * layouts of gdn_frame_forward; they need no alignment. Page-locked (pinned) host memory lets
 * the copies run asynchronously and overlap; pageable memory works but serialises them.
 * The clip is streamed through the GPU in segments of frames (GDN_HOST_SEGMENT_FRAMES frames,
 * read on every call; default about 256 MB of q/k/v per segment): while segment i is computed
 * on `stream`, segment i+1's inputs are copied in and segment i-1's output is copied out on two
 * internal copy streams, ordered by events, through two device staging buffers. The state is
 * carried on the device between segments, so the result is that of gdn_frame_forward over the
 * whole clip, computed as a clip resumed at the segment boundaries (same values up to the
 * rounding of the bf16 copies of S).
 * Asynchronous: when `stream` completes, out and state_out hold the result and the inputs may
 * be reused; read them only after synchronising `stream`. Device memory: two staging buffers of
 * one segment each (cached per GPU and grown on demand like the workspace) plus the workspace of
 * one segment's forward. Host-side errors are returned before anything is enqueued; an error
 * while enqueuing leaves the earlier segments enqueued.
 */
gdn_status gdn_frame_forward_host(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                  const float* gamma, const float* beta, const float* state_in,
                                  gdn_bf16* out, float* state_out, int B, int H, int T, int N,
                                  int D, float key_scale, gdn_stream_t stream);

/*
 * gdn_frame_forward_noalloc - gdn_frame_forward for callers that must not allocate device memory.
 * (No counterpart in the paper: this is a deployment variant of the same computation.)
 *
 * Some callers cannot let a library call cudaMalloc: code inside an inference server or host
 * framework that owns all device memory through its own pool (an allocation behind its back
 * breaks its accounting and can fail or fragment), real-time loops where the device-wide
 * synchronisation that growing gdn_frame_forward's workspace implies would stall other streams,
 * and plugins whose memory budget is fixed when they are loaded. This entry point allocates
 * nothing: its scratch is a fixed 64 MiB array in device memory that the library reserves on
 * every GPU that loads it, held until the process exits.
 *
 * Arguments, layouts and results are exactly those of gdn_frame_forward; the caller still
 * provides q, k, v, gamma, beta, state_in, out and state_out. Limits and behaviour:
 *  - The problem must fit the scratch: the three-kernel workspace (A_t, B_t and S_t of every
 *    frame-head, 128 KiB each at D = 128) must be at most 64 MiB (for D = 128 that is
 *    B*H*T <= 512 frame-heads). Larger problems return GDN_ERR_SCRATCH_LIMIT before
 *    anything is launched.
 *  - The first call on each GPU looks up the scratch's device address (with that GPU current) and
 *    caches it; make that first call before any stream capture.
 *  - All calls on a GPU share the one scratch array, which keeps the last call's contents (no call
 *    needs it cleared: every element is written before it is read). Calls whose executions
 *    overlap on the GPU (different streams, or different host threads) race on it.
 */
gdn_status gdn_frame_forward_noalloc(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                     const float* gamma, const float* beta,
                                     const float* state_in, gdn_bf16* out, float* state_out,
                                     int B, int H, int T, int N, int D, float key_scale,
                                     gdn_stream_t stream);

/*
 * gdn_frame_step - one streaming step: one new frame per stream, carried state.
 * q, k, v, out: [B, N, H, D] bf16; gamma, beta: [B, H] f32; state_in, state_out:
 * [B, H, D, D] f32 (state_in may be NULL for S_0 = 0; state_out == state_in is allowed and is
 * the usual streaming call). Equivalent to gdn_frame_forward with T = 1 (the chunk-causal and
 * distilled autoregressive inference modes advance the state one latent frame at a time:
 * gen-hub.ru SANA-WM article, section "Три режима на любой вкус").
 * For 64 < D <= 128 (and forward mode != 1) one cooperative launch of the step kernel does the
 * whole step in one pass over q, k, v and the state (statistics units and output units taken
 * dynamically); other head dims use the three-kernel path with T = 1. The step kernel keeps a
 * few per-GPU hand-off words (allocated once, zero-initialised) in addition to the workspace.
 */
gdn_status gdn_frame_step(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                          const float* gamma, const float* beta, const float* state_in,
                          gdn_bf16* out, float* state_out, int B, int H, int N, int D,
                          float key_scale, gdn_stream_t stream);

/*
 * gdn_frame_stats - the frame statistics alone, for every frame in parallel:
 *   A_out[b,h,t] = A_t = s^2 K_t^T K_t   as bfloat16, [B, H, T, D, D] (row k', column k)
 *   B_out[b,h,t] = B_t = s   V_t^T K_t   as float32,  [B, H, T, D, D] (row v,  column k)
 * k, v: [B, T, N, H, D] bf16. Both outputs are caller-owned device buffers (no workspace).
 */
gdn_status gdn_frame_stats(const gdn_bf16* k, const gdn_bf16* v, gdn_bf16* A_out, float* B_out,
                           int B, int H, int T, int N, int D, float key_scale,
                           gdn_stream_t stream);

/*
 * gdn_block_causal_la - block-causal linear attention (the predecessor layer: "SANA-Video:
 * Efficient Video Generation with Block Linear Diffusion Transformer", ICLR 2026 oral talk,
 * block KV cache passage -- the D x D state of block i is the cached state of block i-1 plus
 * block i's contribution). Blocks are frames_per_block consecutive frames (the last block may
 * be shorter); every token of block j reads the state after block j:
 *   S += relu(K_j)^T V_j,  z += sum_i relu(k_i),  o = relu(q) S / (relu(q) . z + 1e-6).
 * q, k, v, out: [B, T, N, H, D] bf16. state_in/state_out: [B, H, D, D] f32 in the key-major
 * layout of that formula (row = key index k, column = value index v); z_in/z_out: [B, H, D] f32.
 * Any of state_in, z_in (S_0 = 0, z_0 = 0) and state_out, z_out may be NULL.
 * D must be a multiple of 8 in [8, 120] (one spare column carries the normaliser).
 * Workspace: gdn_la_workspace_bytes(B, H, T, D).
 */
gdn_status gdn_block_causal_la(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                               const float* state_in, const float* z_in, gdn_bf16* out,
                               float* state_out, float* z_out, int B, int H, int T, int N, int D,
                               int frames_per_block, gdn_stream_t stream);

/*
 * gdn_frame_backward - gradients of gdn_frame_forward, for training.
 * (The chatpaper.ai abstract of SANA-WM says the model is trained natively on one-minute
 * clips. The gen-hub.ru article, section "Архитектура", introduces the 1/sqrt(D*S) key scale as
 * a training-stability fix. The pages give no backward; this is the chain rule of the forward.)
 *
 * Given the forward's inputs (q, k, v, gamma, beta, state_in) and the cotangents d_out
 * (dL/dout, [B, T, N, H, D] bf16) and d_state_out (dL/dS_T, [B, H, D, D] f32, NULL = zero),
 * computes dq, dk, dv ([B, T, N, H, D] bf16; dk is the gradient of the UNSCALED keys),
 * d_gamma, d_beta ([B, T, H] f32) and, if d_state_in != NULL, dL/dS_0 ([B, H, D, D] f32).
 * With G_t = dL/dS_t:
 *   G_{T-1} = d_state_out + dO_{T-1}^T Q_{T-1},
 *   G_{t-1} = gamma_t G_t (I - beta_t A_t) + dO_{t-1}^T Q_{t-1},  d_state_in = gamma_0 G_0 (I - beta_0 A_0),
 *   dq_t = dO_t S_t,  dv_t = s beta_t K_t G_t^T,  dk_t = s beta_t (V_t G_t + K_t W'_t),
 *   W'_t = -s gamma_t (S_{t-1}^T G_t + G_t^T S_{t-1}),
 *   d_gamma_t = <G_t, S_{t-1}> - beta_t <G_t, S_{t-1} A_t>,  d_beta_t = <G_t, B_t> - gamma_t <G_t, S_{t-1} A_t>,
 * with s = key_scale, A_t, B_t the forward's frame statistics and S_t the forward's states,
 * which this call recomputes (nothing is kept from a forward call).
 * Steps (7 launches): the forward's statistics and state chain (S_t as bf16), the statistics
 * E_t = dO_t^T Q_t, a reverse state chain for G_t (bf16 copies kept), a per-frame kernel for
 * W'_t, d_gamma, d_beta, and two token passes (dq; dk with dv). When B*H is at most a quarter
 * of the SM count, the E_t statistics, the dq pass and the per-frame and dk/dv passes run on an
 * internal second stream beside the two state chains, the reverse chain in segments of about
 * GDN_BWD_SEGMENT_FRAMES frames (forked from and joined back to `stream` through events, so the
 * call is ordered on `stream` like any other). The first such call on a GPU creates that stream
 * and its events, and sizes the workspace; to capture the call in a CUDA graph, make one
 * uncaptured call with the same sizes first.
 * D must be a multiple of 8 in (64, 128] (GDN_ERR_UNSUPPORTED otherwise). All pointers are
 * device pointers, 16-byte aligned. state_in, d_state_out and d_state_in may be NULL.
 * dq, dk, dv must not overlap each other or q, k, v, d_out; d_gamma, d_beta must not overlap
 * each other or gamma, beta; d_state_in must not overlap state_in (it may alias d_state_out).
 * Workspace: gdn_backward_workspace_bytes(B, H, T, N, D) bytes, about 256 KB per frame-head
 * at D = 128 (the shared per-GPU workspace grows to it).
 */
gdn_status gdn_frame_backward(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                              const float* gamma, const float* beta, const float* state_in,
                              const gdn_bf16* d_out, const float* d_state_out, gdn_bf16* dq,
                              gdn_bf16* dk, gdn_bf16* dv, float* d_gamma, float* d_beta,
                              float* d_state_in, int B, int H, int T, int N, int D,
                              float key_scale, gdn_stream_t stream);

/* Device workspace bytes gdn_frame_backward needs for these sizes. */
size_t gdn_backward_workspace_bytes(int B, int H, int T, int N, int D);

/*
 * Training pair: a forward that keeps what the backward needs, and a backward that uses it
 * instead of recomputing the forward's statistics and state chain (which read k and v again).
 *
 * gdn_frame_forward_train: gdn_frame_forward (same arguments and results; the fused kernel with
 * one ring slot per frame where the fused forward applies, else the three kernels) that also
 * stores, in the caller's device buffer `saved` (gdn_train_saved_bytes(B, H, T, N, D) bytes,
 * 256-byte aligned, not overlapping q, k, v or out), every frame's A_t (bf16), B_t (f32) and
 * S_t (bf16) in the library's internal layout. 64 < D <= 128 (GDN_ERR_UNSUPPORTED otherwise);
 * the buffer's contents are only meaningful to gdn_frame_backward_saved.
 * gdn_frame_backward_saved: gdn_frame_backward (same arguments, results, alignment and overlap
 * rules) for the same q, k, v, gamma, beta, state_in and key_scale that the forward saved, with
 * `saved` read instead of recomputed: it skips one statistics pass over k and v and the forward
 * state chain, and computes dq and the output statistic E_t = dO^T Q in one pass over dO, run
 * ahead of the reverse state chain segment by segment. Results are bit-identical to
 * gdn_frame_backward's. Its workspace is smaller than gdn_frame_backward's (no A_t, B_t, S_t).
 * gdn_train_saved_bytes returns 0 for unsupported sizes.
 */
size_t gdn_train_saved_bytes(int B, int H, int T, int N, int D);
gdn_status gdn_frame_forward_train(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                   const float* gamma, const float* beta, const float* state_in,
                                   gdn_bf16* out, float* state_out, void* saved, int B, int H,
                                   int T, int N, int D, float key_scale, gdn_stream_t stream);
gdn_status gdn_frame_backward_saved(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                    const float* gamma, const float* beta, const float* state_in,
                                    const void* saved, const gdn_bf16* d_out,
                                    const float* d_state_out, gdn_bf16* dq, gdn_bf16* dk,
                                    gdn_bf16* dv, float* d_gamma, float* d_beta,
                                    float* d_state_in, int B, int H, int T, int N, int D,
                                    float key_scale, gdn_stream_t stream);

/*
 * gdn_rope_3d - 3D rotary position embedding of q or k before the attention layers.
 * (The transcript of the ICLR 2026 oral talk "SANA-Video: Efficient Video Generation with Block
 * Linear Diffusion Transformer" introduces a 3D RoPE for the linear attention. The pages give no
 * formula and do not say whether SANA-WM's GDN blocks apply it; the caller decides. The reading
 * below is the plainest one.)
 *
 * x, y: [B, T, N, H, D] bf16 device pointers, 16-byte aligned. y may equal x (in place); any
 * other overlap is rejected. The N tokens of a frame are a grid_h x grid_w latent grid, row-major
 * (token n at row n / grid_w, column n % grid_w). The head dimension splits into three even
 * slices: time d_t, rows d_h and columns d_w, with d_h = d_w = 2 * floor(D / 6) and
 * d_t = D - 2 * d_h (44 / 42 / 42 at D = 128). In each slice of width d, the pairs
 * (x_{2i}, x_{2i+1}) rotate by pos * base^(-2i / d):
 *   (x, y) -> (x cos a - y sin a, x sin a + y cos a).
 * pos is t + t_offset for the time slice (t_offset: absolute index of the clip's first frame, so
 * a streaming step continues a clip), the row for the row slice, the column for the column slice.
 * The angles are computed in double precision, the rotation in f32, and the result is rounded
 * to bf16.
 * D must be a multiple of 8 (GDN_ERR_UNSUPPORTED otherwise). grid_h * grid_w == N, base > 1 and
 * t_offset >= 0 are required (GDN_ERR_INVALID_ARG). Two launches. Workspace: the cos/sin table,
 * 8 * (T * l_t + grid_h * l_h + grid_w * l_w) bytes, from the shared workspace, where l_t, l_h
 * and l_w are the pair counts of the three slices (d_t / 2, d_h / 2, d_w / 2) padded to even row
 * lengths that start on an even pair index (each at most 2 more than its slice's pair count).
 */
gdn_status gdn_rope_3d(const gdn_bf16* x, gdn_bf16* y, int B, int T, int N, int H, int D,
                       int grid_h, int grid_w, float base, int t_offset, gdn_stream_t stream);

/*
 * gdn_softmax_attention - the softmax attention of the hybrid DiT's softmax blocks (the
 * ai-papers.net SANA-WM article, section "ハイブリッドアテンション機構", and the gen-hub.ru article,
 * section "Архитектура: четыре нетривиальных решения": softmax attention in blocks 3, 7, 11, 15
 * and 19 of 20; the same gen-hub.ru article, section "Три режима на любой вкус": bidirectional and
 * chunk-causal autoregressive generation). Per (batch, head), over the clip's T*N tokens:
 *   out = softmax(Q K^T * scale + M) V,
 * where a token of frame t sees every token of the frames t' < (t / F + 1) * F (F =
 * frames_per_chunk): bidirectional inside a chunk of F frames, causal across chunks; F >= T is
 * full bidirectional attention. q and k arrive with any positional encoding already applied.
 * q, k, v, out: [B, T, N, H, D] bf16 device pointers (the layout of the GDN entry points),
 * 16-byte aligned; out must not overlap q, k or v. scale: 0 selects 1/sqrt(D); otherwise finite
 * and > 0. D a multiple of 8 in [8, 128] (GDN_ERR_UNSUPPORTED otherwise); T*N < 2^31.
 * One launch: a persistent tcgen05 kernel (S = Q K^T and O += P V on the tensor cores with
 * accumulators in TMEM, an online softmax with f32 row statistics, P rounded to bf16 for the
 * second product, O / l rounded to bf16) whose CTAs take (batch, head, query tile) items from a
 * work counter, the only workspace it uses (256 bytes of the shared workspace).
 */
gdn_status gdn_softmax_attention(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                 gdn_bf16* out, int B, int H, int T, int N, int D,
                                 int frames_per_chunk, float scale, gdn_stream_t stream);

/* Device workspace bytes gdn_frame_forward / gdn_frame_step need for these sizes. */
size_t gdn_workspace_bytes(int B, int H, int T, int N, int D);
/* Device workspace bytes gdn_block_causal_la needs. */
size_t gdn_la_workspace_bytes(int B, int H, int T, int D);

/* Static description of a status code (never NULL). */
const char* gdn_status_string(gdn_status status);

/*
 * gdn_sync_status - synchronise `stream`, then return and clear the device status word of the
 * current GPU: GDN_OK, GDN_ERR_TIMEOUT if a kernel gave up a bounded wait, or GDN_ERR_CUDA if
 * the synchronisation itself failed.
 */
gdn_status gdn_sync_status(gdn_stream_t stream);

/*
 * Free the cached workspace of the current GPU (synchronises the device first), with the
 * step kernel's hand-off words, the backward's second stream and the host-buffer pipeline's
 * staging buffers and streams. It also forgets what the library cached about the current
 * CUDA context (kernel shared-memory attributes, the device address of
 * gdn_frame_forward_noalloc's scratch), so after a context reset (cudaDeviceReset) call it
 * once, with that GPU current, before the next library call on that GPU.
 */
void gdn_release_workspace(void);

/*
 * Launch profiling (CUDA events around every kernel the library launches).
 * gdn_profile_arm(events, n): from now on, launch i (counted from this call) records
 * events[2i] on its stream just before the kernel and events[2i+1] just after, while
 * 2i+1 < n. events is an array of n cudaEvent_t created by the caller (the library neither
 * creates nor destroys them and keeps the pointer until disarmed); events == NULL disarms.
 * gdn_profile_count(): launches recorded since arming. gdn_profile_kernel(i): the kernel name
 * of recorded launch i ("" if out of range). Not thread-safe against concurrent library calls.
 */
gdn_status gdn_profile_arm(void* const* events, int n);
int gdn_profile_count(void);
const char* gdn_profile_kernel(int i);

/*
 * gdn_set_forward_mode - how gdn_frame_forward / gdn_frame_step run (process-wide):
 *   0 (default) automatic: the chunked forward when an estimate of the per-head state chain's
 *     latency says it pays (few (batch, head) chains over long clips, T >= 16), else the fused
 *     persistent kernel when B*H is at most a third of the SMs and T >= 4, else three kernels
 *     (statistics, state chain, output);
 *   1 always the three kernels;
 *   2 the fused kernel whenever it can run (B*H <= SMs - 8 and cooperative launch available);
 *   3 always the chunked forward: frames are cut into chunks of L (GDN_CHUNK_LEN, else chosen
 *     per problem); each chunk's affine frame maps are composed in parallel (S_end = S_start P_c
 *     + C_c, with P_c the ordered product of gamma_t (I - beta_t A_t) and C_c the accumulated
 *     offset), one scan per head carries the state across chunks, and every chunk then replays
 *     its frames from its start state to produce S_t for the outputs.
 * All compute the same result up to rounding. Returns GDN_ERR_INVALID_ARG for other values.
 */
gdn_status gdn_set_forward_mode(int mode);

/* Library ABI version (major * 100 + minor). */
int gdn_version(void);

/*
 * Debug library (libgdn_debug.so, the same sources built with -DGDN_DEBUG; the stand-in for a
 * memory checker on machines where none can run). Every TMA, bulk and cp.async copy and every
 * tensor-core operand address is checked on the device before it is issued: shared-memory
 * ranges inside the kernel's allocation, the copies' 16-byte alignments and sizes, TMA
 * coordinates (innermost coordinate a multiple of 16 elements, no negative store coordinate).
 * A violation skips the copy (the call then ends on a bounded wait with GDN_ERR_TIMEOUT, never on
 * a fault) and records its site (1 TMA load shared address, 2 TMA load coordinate, 3 TMA store
 * shared address, 4 TMA store coordinate, 5 bulk copy shared range, 6 bulk copy global address
 * or size, 7 cp.async address, 8 MMA operand address) and the offending value.
 * gdn_debug_checks(): 1 in the debug library, 0 in the release library (which compiles the checks
 * out). gdn_debug_report(site, value): synchronous; 1 if a violation was recorded since the last
 * report (site and value filled, the record cleared), 0 if none, -1 on a CUDA error. Either
 * pointer may be NULL.
 */
int gdn_debug_checks(void);
int gdn_debug_report(int* site, long long* value);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
