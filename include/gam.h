/*
 * gam.h -- C ABI of the GigaAM Conformer encoder + CTC hot path on B200 (sm_100a).
 *
 * The path (audio -> log-mel -> Conv1d 4x subsampling -> N Conformer blocks ->
 * CTC head -> greedy collapse) follows these pages:
 *   - "GigaAM v3 MLX", sections "Runtime pipeline", "Frontend configuration"
 *     and "Architecture details";
 *   - "GigaAM on MLX: the transcripts matched, but the model was broken",
 *     sections "What we're porting", "Trap 1" (RoPE base 5000), "Trap 2"
 *     (RoPE on the raw input before linear_q / linear_k), "Trap 3" (stored
 *     window and filterbank) and "Trap 4" (PyTorch weight layouts, fp16);
 *   - "GigaAM v3 RNNT -- MLX (Apple Silicon)", section "Notes for other
 *     runtimes" (center=False, log(clip(x, 1e-9, 1e9)), blank = len(vocab));
 *   - "GigaAM MLX port for Mac", sections "What is inside the model" and
 *     "How precision affects size and speed" (INT8 weights, one scale per
 *     group of 64).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Plain C types only.  "device pointer" means memory the caller allocated
 *   on the context's GPU (cudaMalloc, torch, ...); "host pointer" means CPU
 *   memory.  `stream` is a cudaStream_t passed as void* (NULL = legacy
 *   default stream).  All GPU work of a call is enqueued on that stream; no
 *   call synchronises it except gam_transcribe, gam_device_status and the
 *   profiling calls (gam_profile_reset / gam_profile_read).
 * - The caller owns every buffer it passes.  A context owns its weights and
 *   one workspace sized at creation for (max_batch, max_samples); calls after
 *   gam_create do no device allocation (CUDA-graph replay included, see
 *   gam_graphs_enable).  Small per-call tables go to the device through a
 *   ring of 8 pinned host buffers; a call waits on the host only if the copy
 *   made 8 calls earlier has not run yet.  One context serves one stream at a
 *   time.
 * - Errors are returned, never thrown and never abort the process.  Arguments
 *   are checked before any launch.  An asynchronous device error shows up as
 *   GAM_ERR_CUDA on a later call.  Device-side waits are bounded; a wait that
 *   gives up sets a status word read by gam_device_status
 *   (GAM_ERR_DEVICE_TIMEOUT).
 * - Lengths are host arrays so the host plans every shape without reading
 *   device memory.  A clip of N samples has F = 1 + (N - 320) / 160 mel
 *   frames (center=false), tensor lengths T1 = (F - 1) / 2 + 1 and
 *   T' = (T1 - 1) / 2 + 1 after the two stride-2 convs, and valid lengths
 *   L1 = (F - 1) / 2 and L' = (L1 - 1) / 2 (integer division).  Every clip
 *   needs L' >= 1, i.e. N >= 1280 samples, else GAM_ERR_SHAPE.
 * - Batched outputs are right-padded: frames at or beyond a clip's length are
 *   written as zeros (token ids as -1).
 */
#ifndef GAM_H
#define GAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GAM_OK = 0,
  GAM_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, non-positive size   */
  GAM_ERR_SHAPE = 2,              /* a clip too short / inconsistent sizes        */
  GAM_ERR_CAPACITY = 3,           /* batch or samples above the context's limits  */
  GAM_ERR_WEIGHTS = 4,            /* missing tensor, wrong shape or dtype         */
  GAM_ERR_UNSUPPORTED_DEVICE = 5, /* not a compute capability 10.0 GPU           */
  GAM_ERR_CUDA = 6,               /* a CUDA runtime / driver call failed          */
  GAM_ERR_DEVICE_TIMEOUT = 7      /* a bounded device-side wait gave up           */
} gam_status;

/* gam_config.precision.  The quantised modes store the linear weights of the
 * encoder blocks and the CTC head as integers q with one fp16 scale s per group
 * of 64 consecutive input weights (w = q s): INT8 q in [-127, 127], INT6 in
 * [-31, 31], INT4 in [-7, 7] ("GigaAM MLX port for Mac", "How precision affects
 * size and speed": INT8, INT6 and INT4 with group 64).  The weights are
 * dequantised to fp16 inside the tensor-core GEMM's mainloop. */
enum { GAM_FP32 = 0, GAM_FP16 = 1, GAM_INT8_G64 = 2, GAM_INT6_G64 = 3, GAM_INT4_G64 = 4 };

/* gam_tensor.dtype */
enum { GAM_DTYPE_F32 = 0, GAM_DTYPE_F16 = 1, GAM_DTYPE_I8 = 2 };

/* Stage ids of gam_encode_stage (the residual stream after each step). */
enum {
  GAM_STAGE_SUBSAMPLING = 0, /* layer ignored: output of the two convs      */
  GAM_STAGE_FFN1 = 1,        /* x + 1/2 FFN1(LN x)                          */
  GAM_STAGE_MHSA = 2,        /* + rotary MHSA                               */
  GAM_STAGE_CONV = 3,        /* + convolution module                        */
  GAM_STAGE_FFN2 = 4,        /* + 1/2 FFN2                                  */
  GAM_STAGE_LAYER = 5        /* block output after its final LayerNorm      */
};

/* Model and capacity.  Field names follow the pages' notation. */
typedef struct {
  int n_layers;      /* Conformer blocks (16 for v3, 24 multilingual large)   */
  int d_model;       /* model width d (768 / 1024); d % 256 == 0              */
  int n_heads;       /* H; d_head = d / H must be 48 or 64                    */
  int ffn_dim;       /* FFN hidden width (4 d); % 256 == 0                    */
  int conv_kernel;   /* depthwise kernel K_dw (odd, <= 63)                    */
  int n_mels;        /* 64                                                    */
  int n_fft;         /* 320                                                   */
  int win;           /* 320                                                   */
  int hop;           /* 160                                                   */
  int sub_kernel;    /* subsampling Conv1d kernel, 5 (stride 2, padding 2)    */
  int n_classes;     /* vocabulary + 1; blank id = n_classes - 1; <= 1024     */
  float rope_base;   /* 5000 (pos_emb_max_len), not 10000                     */
  float ln_eps;      /* LayerNorm eps (1e-5)                                  */
  float bn_eps;      /* BatchNorm eps (1e-5)                                  */
  int precision;     /* GAM_FP32, GAM_FP16, GAM_INT8_G64, GAM_INT6_G64, GAM_INT4_G64 */
  int max_batch;     /* capacity: clips per call                              */
  int64_t max_samples; /* capacity: samples per clip                          */
} gam_config;

/* One named weight tensor, HOST memory, PyTorch layout (Linear [out, in],
 * Conv1d [out, in, K]).  gam_create copies it; the caller may free it after. */
typedef struct {
  const char* name;
  const void* data;
  int dtype;         /* GAM_DTYPE_*                                           */
  int ndim;
  int64_t shape[4];
} gam_tensor;

typedef struct gam_ctx gam_ctx;

/* Human-readable name of a status code (static storage). */
const char* gam_status_string(gam_status status);

/* Text of the last error seen by this context ("" if none).  A NULL ctx gives
 * the last error on this thread of the calls that take no context
 * (gam_create, gam_plan_lengths, gam_ctc_collapse_noalloc). */
const char* gam_last_error(const gam_ctx* ctx);

/* Lengths of the frontend and subsampling ("GigaAM v3 MLX", "Frontend
 * configuration": window 320, hop 160, center false; "Validation" prints a
 * 1 s clip as [64, 99] features and [1, 768, 25] encoder output).
 * Host-only length planning for `batch` clips of `lengths_host[i]` samples.
 * Writes (each optional, may be NULL) frames_out[i] = F_i, enc_len_out[i] =
 * L'_i, and dims_out[0..1] = (F_max, T'_max), the padded sizes of the mel and
 * encoder outputs.  Fails with GAM_ERR_SHAPE for a clip shorter than 1280. */
gam_status gam_plan_lengths(const gam_config* cfg, const int32_t* lengths_host, int batch,
                            int32_t* frames_out, int32_t* enc_len_out, int32_t* dims_out);

/* Model setup ("GigaAM on MLX: the transcripts matched, but the model was
 * broken", "Trap 3" (the stored window and filterbank are inputs) and "Trap 4"
 * (PyTorch weight layouts, fp16 checkpoints); "GigaAM v3 MLX",
 * "Architecture details"; "GigaAM MLX port for Mac", "How precision affects
 * size and speed" (one scale per group of 64 weights).
 * Build a context on CUDA device `device`: checks the device (sm_100),
 * validates every tensor the config needs by name/shape/dtype, repacks the
 * weights (fold the window into a DFT basis, fold BatchNorm into the depthwise
 * conv, reorder GLU halves, transpose conv weights, quantised layouts), and
 * allocates the workspace.  Tensors: "frontend.window" [win] f32,
 * "frontend.mel_fb" [n_fft/2+1, n_mels] f32, "subsampling.conv{1,2}.{weight,
 * bias}", per layer l "layers.l.{ffn1,ffn2}.{norm,linear1,linear2}.*",
 * "layers.l.attn.{norm,linear_q,linear_k,linear_v,linear_out}.*",
 * "layers.l.conv.{norm,pointwise1,depthwise,bn,pointwise2}.*",
 * "layers.l.norm_out.*", "head.{weight,bias}" ([C, d] or [C, d, 1]).  In
 * the quantised precisions the eleven linear weights of a block and the head's
 * are given as "<name>.weight_q" (int8 array of the weight's shape holding q,
 * within the precision's range, else GAM_ERR_WEIGHTS) and "<name>.weight_scale"
 * (f16 [out, in/64]); all other tensors f16 or f32.  6- and 4-bit weights are
 * packed on the device at 6 and 4 bits per weight.  On success *out owns
 * device memory until gam_destroy.  The environment variable GAM_GEMM_TILES
 * (read here) sets the tile policy of the fp16 tensor-core GEMMs: "single"
 * (single-CTA tiles only), "pair" (paired-CTA tiles wherever one applies) or,
 * by default, "auto" (the cheaper of the two by the library's cost model).
 * The encoder's kernels are launched with programmatic dependent launch (each
 * kernel's setup overlaps the previous kernel's tail; data order unchanged);
 * GAM_PDL=0 in the environment turns that off. */
gam_status gam_create(const gam_config* cfg, const gam_tensor* tensors, int n_tensors, int device,
                      gam_ctx** out);

/* Free everything the context owns.  NULL is accepted. */
gam_status gam_destroy(gam_ctx* ctx);

/* Log-mel frontend only ("GigaAM v3 MLX", "Frontend configuration").
 * audio_dev: device f32 [batch, max_samples] (row stride max_samples), clip i
 * valid on its first lengths_host[i] samples.  mel_dev: device f32
 * [batch, F_max, n_mels], time-major (the pages print [n_mels, F]); frames at
 * or beyond F_i are zero.  frames_host_out (optional): F_i. */
gam_status gam_logmel(gam_ctx* ctx, const float* audio_dev, const int32_t* lengths_host, int batch,
                      int64_t max_samples, float* mel_dev, int32_t* frames_host_out, void* stream);

/* The encoder ("GigaAM v3 MLX", "Runtime pipeline" and "Architecture
 * details"; the Russian original of "GigaAM MLX port for Mac", pipeline list
 * under "What is inside the model": log-mel -> two Conv1d layers -> Conformer
 * blocks of FFN, attention, convolution, FFN; RoPE per "GigaAM on MLX ...",
 * "Trap 1" and "Trap 2").
 * Frontend + subsampling + all Conformer blocks.  enc_dev: device f32
 * [batch, T'_max, d]; frames at or beyond L'_i are zero.  enc_len_host_out
 * (optional): L'_i. */
gam_status gam_encode(gam_ctx* ctx, const float* audio_dev, const int32_t* lengths_host, int batch,
                      int64_t max_samples, float* enc_dev, int32_t* enc_len_host_out, void* stream);

/* Debug tap for layer-by-layer localisation ("GigaAM on MLX ...", "Trap 1"):
 * runs the same path as gam_encode up to `stage` of block `layer` and writes
 * the f32 residual stream there to out_dev [batch, T'_max, d] (zero padded). */
gam_status gam_encode_stage(gam_ctx* ctx, const float* audio_dev, const int32_t* lengths_host, int batch,
                            int64_t max_samples, int layer, int stage, float* out_dev, void* stream);

/* CTC head + greedy decoding (the Russian original of "GigaAM MLX port for
 * Mac", pipeline list under "What is inside the model": a CTC layer gives each
 * symbol's probability per step, decoding removes repeats and blanks; blank =
 * len(vocabulary) per "GigaAM v3 RNNT -- MLX (Apple Silicon)", "Notes for
 * other runtimes").
 * enc_dev: device f32 [batch, t_max, d] with
 * clip i valid on its first enc_len_host[i] <= t_max frames.  logp_dev
 * (optional, device f32 [batch, t_max, n_classes]): log-softmax of the head's
 * logits, zero beyond a clip.  tokens_dev: device i32 [batch, t_max], the
 * collapsed ids (runs merged, then blanks dropped; argmax = lowest index of
 * the fp32 maximum), -1 after the last token.  counts_dev: device i32 [batch].
 * The argmax follows numpy's order: a NaN logit ranks above every number (the
 * first NaN wins) and a frame whose logits are all equal, all -inf included,
 * gives index 0; such frames have NaN log-probabilities. */
gam_status gam_ctc_greedy(gam_ctx* ctx, const float* enc_dev, const int32_t* enc_len_host, int batch,
                          int t_max, float* logp_dev, int32_t* tokens_dev, int32_t* counts_dev,
                          void* stream);

/* gam_ctc_greedy with each token's position: frames_dev device i32 [batch,
 * t_max] receives the encoder frame where the token's run of equal argmax
 * values starts (-1 after the last token), which places the token in time for
 * joining the transcripts of overlapping long-form chunks ("GigaAM v3 MLX",
 * "Long-form transcription": 20 s chunks, 0-2 s overlap).  No log-probs. */
gam_status gam_ctc_greedy_frames(gam_ctx* ctx, const float* enc_dev, const int32_t* enc_len_host, int batch,
                                 int t_max, int32_t* tokens_dev, int32_t* frames_dev, int32_t* counts_dev,
                                 void* stream);

/* Greedy decoding from given scores, the decoding step of gam_ctc_greedy on
 * its own (same passages as gam_ctc_greedy):
 * logits_dev device f32 [batch, t_max, n_classes]; blank = n_classes - 1;
 * outputs as gam_ctc_greedy.  Uses the context's workspace for the per-frame
 * argmax, so batch * t_max must fit its capacity. */
gam_status gam_ctc_collapse(gam_ctx* ctx, const float* logits_dev, const int32_t* lengths_host, int batch,
                            int t_max, int n_classes, int32_t* tokens_dev, int32_t* counts_dev, void* stream);

/* End-to-end call on HOST buffers: copies audio_host [batch, max_samples] f32
 * to the device, runs gam_encode and gam_ctc_greedy, copies tokens_host
 * [batch, T'_max] and counts_host [batch] back, and synchronises `stream`
 * before returning.  Pinned host memory makes the copies asynchronous. */
gam_status gam_transcribe(gam_ctx* ctx, const float* audio_host, const int32_t* lengths_host, int batch,
                          int64_t max_samples, int32_t* tokens_host, int32_t* counts_host, void* stream);

/* Synchronises the context's last stream and reports GAM_ERR_DEVICE_TIMEOUT
 * if a device-side bounded wait gave up since the last gam_profile_reset. */
gam_status gam_device_status(gam_ctx* ctx);

/* ---- profiling (per kernel family, CUDA events on the launching stream) ---- */

/* Choose which kernel families get an event pair recorded around every
 * launch: 0 = none, -1 = all, else a bit mask (bit k = family k).  Each
 * timed launch costs about a microsecond of stream time.  Resets the counters. */
gam_status gam_profile_enable(gam_ctx* ctx, int on);
gam_status gam_profile_reset(gam_ctx* ctx);
/* Number of kernel families and the name of family `kind`. */
int gam_profile_kinds(void);
const char* gam_profile_kind_name(int kind);
/* Totals since the last reset for family `kind` (synchronises the recorded
 * events).  Launch counts are kept even when timing is off. */
gam_status gam_profile_read(gam_ctx* ctx, int kind, double* total_ms, int64_t* launches);

/* ---- RNNT head ---- */

/* RNNT head of the v3 RNNT and E2E RNNT models ("GigaAM on MLX: the
 * transcripts matched, but the model was broken", "What we're porting": a
 * single-layer LSTM of size 320 plus a joint network; "Trap 4" and "GigaAM v3
 * RNNT -- MLX (Apple Silicon)", "Notes for other runtimes": PyTorch LSTM
 * weights, bias = bias_ih + bias_hh, blank = len(vocabulary); "GigaAM v3 MLX",
 * "Architecture details": greedy RNNT decoding, 1025 classes with blank 1024). */
typedef struct {
  int n_classes;    /* vocabulary + 1; blank = n_classes - 1 (34 or 1025); <= 4096        */
  int pred_dim;     /* LSTM hidden size P (320), a multiple of 8                           */
  int joint_dim;    /* joint hidden width J (320), a multiple of 8                         */
  int max_symbols;  /* symbols emitted per encoder frame at most (10), 1..64               */
  int joint_act;    /* 0: ReLU, 1: tanh, applied to W_enc f + b_enc + W_pred g + b_pred     */
} gam_rnnt_config;

/* Attach an RNNT head to a context (once).  Tensors, HOST memory, f16 or f32,
 * PyTorch layout: "rnnt.embed.weight" [C, E], "rnnt.lstm.weight_ih_l0"
 * [4P, E], "rnnt.lstm.weight_hh_l0" [4P, P], "rnnt.lstm.bias_ih_l0" and
 * "rnnt.lstm.bias_hh_l0" [4P] (gate order i, f, g, o), "rnnt.joint.enc.weight"
 * [J, d_model], "rnnt.joint.enc.bias" [J], "rnnt.joint.pred.weight" [J, P],
 * "rnnt.joint.pred.bias" [J], "rnnt.joint.out.weight" [C, J],
 * "rnnt.joint.out.bias" [C].  The head's weights stay fp16 / fp32 in every
 * precision.  Allocates device memory (weights, a per-symbol table of the
 * LSTM's input gates and a projection buffer for max_batch clips) and
 * synchronises the device once. */
gam_status gam_rnnt_attach(gam_ctx* ctx, const gam_rnnt_config* cfg, const gam_tensor* tensors, int n_tensors);

/* Greedy RNNT decoding of encoder output.  enc_dev: device f32 [batch, t_max,
 * d] (gam_encode's output), clip i valid on its first enc_len_host[i] frames.
 * The predictor starts from a zero input and zero state and takes the
 * embedding of each emitted symbol; at frame t the decoder repeats {joint
 * logits = W_out act(W_enc f_t + b_enc + W_pred g + b_pred) + b_out; argmax,
 * lowest index on ties; blank -> next frame, else emit} with at most
 * max_symbols symbols per frame.  tokens_dev device i32 [batch, max_tokens]:
 * the symbols, -1 after the last; frames_dev (optional, device i32 [batch,
 * max_tokens]): the encoder frame of each symbol, -1 after the last;
 * counts_dev device i32 [batch]: symbols stored (at most max_tokens; symbols
 * past max_tokens are decoded but not stored, and t_max * max_symbols never
 * loses any).  The encoder half of the joint is one tensor-core GEMM over all
 * valid frames; the loop is one kernel, by default a cluster of 8 CTAs per clip
 * holding the head's weights in shared memory; heads whose weight slices do not
 * fit (e.g. 4096 classes or a 1024-wide predictor) stream the weights through
 * one CTA per clip instead, and GAM_RNNT=ring in the environment forces that
 * form.  Clips with more decisions take longer; the call's time is that of the
 * slowest clip. */
gam_status gam_rnnt_greedy(gam_ctx* ctx, const float* enc_dev, const int32_t* enc_len_host, int batch, int t_max,
                           int max_tokens, int32_t* tokens_dev, int32_t* frames_dev, int32_t* counts_dev,
                           void* stream);

/* ---- pseudo-streaming ---- */

/* Pseudo-streaming as "GigaAM on MLX: the transcripts matched, but the model
 * was broken", "Streaming" describes it: the model is not a streaming model, so
 * every step re-recognises the audio received so far, but no more than the
 * last window_samples (30 s = 480000 samples there).  A gam_stream belongs to
 * one context and allocates its buffers at creation (two window buffers, the
 * encoder output and tokens of one window); pushes allocate nothing.  Once the
 * window is full, every push encodes the same length from one of two buffers,
 * so the context's CUDA graphs replay from the fourth push on. */
typedef struct gam_stream gam_stream;

/* window_samples: 1280 .. the context's max_samples (GAM_ERR_CAPACITY). */
gam_status gam_stream_create(gam_ctx* ctx, int64_t window_samples, gam_stream** out);
gam_status gam_stream_destroy(gam_stream* st);
/* Forget the audio pushed so far. */
gam_status gam_stream_reset(gam_stream* st);

/* Append n samples (HOST f32, 16 kHz mono) and recognise the window, i.e. the
 * last min(total, window_samples) samples: gam_encode + gam_ctc_greedy of that
 * window as one clip, on `stream`, synchronised before returning.
 * tokens_host receives the window's CTC tokens (at most max_tokens of them),
 * *count_out the window's token count (possibly above max_tokens), and
 * *window_start_out (optional) the index of the window's first sample in the
 * pushed stream.  A window shorter than 1280 samples has no encoder frame and
 * gives 0 tokens.  The tokens of a step are the whole window's transcript, not
 * only the new part: as the page notes, the cost of a step grows with the
 * window, and text at its start can change from step to step. */
gam_status gam_stream_push(gam_stream* st, const float* samples_host, int64_t n, int32_t* tokens_host,
                           int max_tokens, int32_t* count_out, int64_t* window_start_out, void* stream);

/* ---- greedy decoding without any allocation ---- */

/* Frames of the fixed scratch array behind gam_ctc_collapse_noalloc. */
#define GAM_NOALLOC_MAX_FRAMES (1 << 20)

/* The pages have no counterpart of this call: it is a service for callers
 * that must not allocate device memory -- code that cannot afford the device
 * synchronisation a cudaMalloc may cause, plug-ins whose host framework owns
 * all device memory, or callers without a gam_ctx.  Same result as
 * gam_ctc_collapse (argmax = lowest index of the fp32 maximum, runs merged,
 * then blanks dropped; tokens -1 after the last one), but it takes no context
 * and allocates nothing: the per-frame argmax it needs lives in a file-scope
 * device array of GAM_NOALLOC_MAX_FRAMES ints (4 MiB) that every GPU loading
 * the library keeps until the process exits.
 *   logits_dev  device f32 [batch, t_max, n_classes]; blank = n_classes - 1
 *   lengths_dev device i32 [batch]: valid frames per clip, clamped to [0, t_max]
 *   tokens_dev  device i32 [batch, t_max]; counts_dev device i32 [batch]
 * batch * t_max above GAM_NOALLOC_MAX_FRAMES fails with GAM_ERR_CAPACITY
 * before any launch (text in gam_last_error(NULL)).  The first call on a
 * device (that device current) looks up the array's device address once and
 * keeps it with the device's current CUDA context; a call that finds another
 * context current (after cudaDeviceReset) looks it up again.  Make the first
 * call on a device before any stream capture.  All calls on a device
 * share the array and each fully rewrites the part it reads, so nothing needs
 * clearing, but calls whose GPU work overlaps (other streams or threads) race
 * on it.  Runs on the current device and on `stream`. */
gam_status gam_ctc_collapse_noalloc(const float* logits_dev, const int32_t* lengths_dev, int batch, int t_max,
                                    int n_classes, int32_t* tokens_dev, int32_t* counts_dev, void* stream);

/* ---- CUDA graphs ---- */

/* Repeated calls of gam_encode, gam_encode_stage and gam_ctc_greedy with the
 * same clip lengths and the same buffer pointers replay a CUDA graph of the
 * call's kernel sequence: the first such call runs eagerly, the second is
 * captured (on a private stream created with the context) and launched on
 * `stream`, later ones are one graph launch.  Each graph reads its clip table
 * from one of 16 device slots allocated by gam_create; the table is copied
 * into its slot asynchronously on `stream` (after the slot's previous graph
 * has finished its last replay), so capturing and evicting allocate no device
 * memory and do not synchronise.  Buffer contents may change between calls;
 * pointers and lengths may not (a different pointer or length is a different
 * graph, up to 16 are kept, least recently used first out; the driver frees
 * an evicted graph once its last replay is done).  No graph is used while
 * profiling is enabled (gam_profile_enable) or an error is injected.  On by
 * default; the environment variable GAM_CUDA_GRAPHS=0 (read by gam_create) or
 * on = 0 here turns it off.  Outputs are bit-identical either way. */
gam_status gam_graphs_enable(gam_ctx* ctx, int on);

/* ---- kernel unit test (tests) ---- */

/* One GEMM of the encoder's kind through the chosen implementation:
 * out[M, N] (device f32, row stride ldo) += A[M, K] . W[N, K]^T + bias[N],
 * where A (row stride lda) and W are device fp16 and bias device f32.
 * impl = kind | (width << 8).  kind 0 = tensor cores (tcgen05) with the tile
 * shape the encoder would choose, 1 = CUDA cores, 2 = tensor cores with
 * single-CTA tiles (128 rows), 3 = tensor cores with paired-CTA tiles (256
 * rows on two SMs, cta_group::2); width 0 lets the library choose the tile
 * width, else 128, 192 or 256 output columns, or 64 with single-CTA tiles of at
 * most 256 rows (tensor-core kinds only; the library picks 64 for such few rows
 * so that more SMs share the weight stream); 4 = tensor cores with K split over
 * a cluster of 2 to 4 CTAs whose partial sums the first CTA adds in a fixed
 * order (at most 256 rows, lda >= k, width 0; the library also picks this for
 * such few rows when K is deep enough to leave each CTA at least 8 k-blocks of
 * 64; GAM_ERR_SHAPE, or GAM_ERR_CUDA when no split count applies to the shape).
 * N % 256 == 0 and K % 64 == 0 for the tensor-core kinds, N % 128 == 0 and
 * K % 16 == 0 for CUDA cores; a width that does not divide N fails with
 * GAM_ERR_SHAPE, an impl outside these values with GAM_ERR_INVALID_ARG.
 * lda < k selects the strided convolution view of the subsampling convs: row
 * r of A is rows 2r .. 2r+k/C-1 of a [rows, C] buffer with lda = 2C
 * (C % 64 == 0), and the buffer must hold (m + 2) * lda elements.  Uses the
 * residual-update epilogue of the encoder (alpha 1). */
gam_status gam_debug_gemm(gam_ctx* ctx, int impl, const void* a_dev, int lda, const void* w_dev,
                          const float* bias_dev, int m, int n, int k, float* out_dev, int ldo, void* stream);

/* ---- bounded device waits (tests) ---- */

/* Test hook for the bounded waits of the tensor-core GEMM.  Applies to the
 * next tensor-core GEMM this context launches (gam_debug_gemm with impl kind 2
 * is the intended one), then switches itself off: that launch's waits give up
 * after limit_ns nanoseconds (> 0) instead of 2 s, and, when skip_k_block >= 0,
 * its producer does not issue the loads of its skip_k_block-th k-block, so the
 * MMA issuer's wait for that stage runs out.  The kernel then drains what is in
 * flight, frees its tensor memory and returns; gam_device_status reports
 * GAM_ERR_DEVICE_TIMEOUT until gam_profile_reset, and the context stays usable.
 * Nothing faults or hangs: every wait involved is bounded. */
gam_status gam_debug_wait_timeout(gam_ctx* ctx, int64_t limit_ns, int skip_k_block);

/* ---- host-side fault injection (tests) ---- */

/* Make the next `count` CUDA-error checks of this context report
 * `cuda_error` (a cudaError_t value) as if the runtime had returned it. */
gam_status gam_debug_inject_cuda_error(gam_ctx* ctx, int cuda_error, int count);

#ifdef __cplusplus
}
#endif

#endif /* GAM_H */
