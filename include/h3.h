/*
 * h3.h -- C ABI of the B200 (sm_100a) H3-Omni block step.
 *
 * One forward pass of the single-stream H3-Omni-Transformer block over a
 * packed text + audio + video token sequence, plus the flow-sampler Euler
 * step.  Sources (page title, section):
 *   [shouss] "MiniMax-H3: native joint audio-video generation"
 *            (note.shouss.top): §2.2 packed sequence, §3 trunk with modality
 *            modulation, §3.1 three modulation groups (6D per modality, 18D
 *            total), §3.2 config table, Q/K RMSNorm then RoPE, SiLU(gate)*up,
 *            §4.1 patch width, §4.3 AudioVAE, §5 non-causal attention and
 *            update mask, §6 velocity sampling with video/audio schedulers.
 *   [gojay]  "MiniMax-H3 paper reading" (gojay.top): §4 f16t4d24 VAE and
 *            1x2x2 patchify, §5 Omni-Transformer, §7.3 shapes, §7.4 3-D
 *            MM-RoPE (audio on the time axis only).
 *   [0539]   "H3's omni-modal ambition" (0539edu.com): scheduler sigma
 *            shifts 12.0 (video) and 3.0 (audio).
 *
 * Conventions (all entry points):
 *   - Tensor arguments are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or synchronises device memory; every call is
 *     asynchronous on the caller's stream (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).
 *   - bf16 tensors are passed as h3_bf16 (the 16-bit pattern).  Weights are
 *     row-major [out, in]; activations are row-major, one token per row.
 *   - Every call validates all arguments before launching anything and
 *     returns H3_OK or a negative status; on error nothing is launched and
 *     h3_last_error() (per host thread) describes the problem.
 *   - Pointers must be 16-byte aligned.  L_pad must be a multiple of 128.
 *   - Modality ids / range order: text = 0, audio = 1, video = 2 (the packing
 *     order text -> audio -> target video -> padding of [shouss] §2.2).
 *   - Residual stream x: fp32 [L_pad][D]; rows >= L are padding (zero).
 *   - Modulation mod: fp32 [3][6][D], per modality (shift_msa, scale_msa,
 *     gate_msa, shift_mlp, scale_mlp, gate_mlp) ([shouss] §3.1).
 */
#ifndef H3_H
#define H3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t h3_bf16;

enum h3_status {
  H3_OK = 0,
  H3_ERR_NULL = -1,        /* a required pointer is NULL */
  H3_ERR_SHAPE = -2,       /* inconsistent sizes or ranges */
  H3_ERR_ALIGN = -3,       /* pointer not 16-byte aligned */
  H3_ERR_UNSUPPORTED = -4, /* head_dim != 128, D % 64 != 0, F % 128 != 0, ... */
  H3_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed */
  H3_ERR_TIMEOUT = -6,     /* a device-side wait gave up (see h3_device_status) */
  H3_ERR_BOUND = -7        /* attention with its norm and RoPE in the prologue met scores
                              outside its static bound (see h3_attention, h3_device_status) */
};

enum h3_modality { H3_TEXT = 0, H3_AUDIO = 1, H3_VIDEO = 2 };
enum h3_branch { H3_MSA = 0, H3_MLP = 1 };

/* h3_qkv_qknorm_mrope / h3_attention flag: Q/K RMSNorm and RoPE are applied
 * in the QKV GEMM epilogue (once per token), and h3_attention consumes the
 * already-rotated q, k (the library's default placement, the faster one).
 * Without it on both calls, the QKV call writes q, k raw and h3_attention
 * applies the norm and RoPE in its prologue: each Q tile once per CTA and
 * each K tile as it lands in shared memory ([shouss] §3.2 fixes the order,
 * norm then RoPE, not the kernel that takes them).  The two placements give
 * the same result up to the bf16 rounding of the raw q, k. */
#define H3_QK_NORM_ROPE_IN_QKV 1
/* With h3_qkv_qknorm_mrope_e4m3 / h3_attention / h3_block_forward_e4m3 only:
 * q and k are passed between the QKV call and attention as e4m3 codes (see
 * the FP8 section), and attention takes S = Q K^T on e4m3 tensor-core MMAs.
 * P V stays bf16. */
#define H3_QK_E4M3 2

/* Block dimensions.  head_dim must be 128; I = H * head_dim;
 * rope_t + rope_h + rope_w = head_dim, each even ([gojay] §7.4).
 * theta: RoPE base (10000); eps_ln: LayerNorm epsilon; eps_qk: Q/K RMSNorm
 * epsilon. */
typedef struct h3_dims {
  int D, H, head_dim, I, F;
  int rope_t, rope_h, rope_w;
  float theta, eps_ln, eps_qk;
} h3_dims;

/* Packed-sequence ranges: rows [start[m], start[m] + count[m]) hold modality
 * m; the three ranges tile [0, L) without overlap ([shouss] §2.2); L_pad is
 * a multiple of 128 with L <= L_pad (h3_make_ranges gives L rounded up; a
 * sequence-parallel shard, h3_sp_make_layout, may pad further). */
typedef struct h3_ranges {
  int start[3];
  int count[3];
  int L;
  int L_pad;
} h3_ranges;

/* Description of the last error on this host thread (never NULL). */
const char* h3_last_error(void);

/* ABI version (major * 100 + minor). */
int h3_version(void);

/* Host only.  Fill `out` for n_text text tokens, n_audio_tokens audio tokens
 * (channels x latents, channel-major) and n_video_tokens video tokens packed
 * text -> audio -> video, L_pad = ceil(L / 128) * 128 ([shouss] §2.2). */
int h3_make_ranges(int n_text, int n_audio_tokens, int n_video_tokens, h3_ranges* out);

/* Host only.  n_steps + 1 sigmas from 1 to 0, uniform then time-shifted,
 * sigma' = shift * sigma / (1 + (shift - 1) * sigma) (video shift 12.0,
 * audio shift 3.0: [shouss] §6, [0539]).  out: host float[n_steps + 1]. */
int h3_sigma_schedule(int n_steps, float shift, float* out);

/* A1 + A2.  Patchify the video latent (1x2x2 over (t, h, w): token (t, i, j)
 * takes latent pixels (t, 2i+ph, 2j+pw), feature (ph*2 + pw)*C_lat + c,
 * [gojay] §4, §7.3), write token positions and modality ids, and project
 * every modality into the residual stream with its own input projection
 * ([gojay] §5: modality-specific parameters only in the I/O layers).
 *   text     [count[TEXT]][D_text]               bf16
 *   video    [T][Hl][Wl][C_lat] channels-last     bf16 (Hl, Wl even; C_lat % 4 == 0)
 *   audio    [audio_channels][n_audio][C_audio]   bf16 (token = ch * n_audio + k)
 *   W_text [D][D_text], W_vid [D][4*C_lat], W_aud [D][C_audio]  bf16
 *   patches  workspace [count[VIDEO]][4*C_lat]     bf16 (caller-owned scratch;
 *            holds the patch rows afterwards)
 *   x_out    [L_pad][D] fp32 (rows >= L zeroed)
 *   pos_out  [L_pad][3] fp32: video (t, i, j); audio latent k at (6k/40, 0, 0),
 *            the 24/4 Hz video-latent time axis shared with 40 Hz audio
 *            ([gojay] §7.4); text and padding (0, 0, 0)
 *   mod_out  [L_pad] uint8 modality id, 255 for padding
 * Requires count[VIDEO] == T * (Hl/2) * (Wl/2) and
 * count[AUDIO] == audio_channels * n_audio. */
int h3_embed_pack(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* text, int D_text,
                  const h3_bf16* video, int T, int Hl, int Wl, int C_lat, const h3_bf16* audio,
                  int audio_channels, int n_audio, int C_audio, const h3_bf16* W_text, const h3_bf16* W_vid,
                  const h3_bf16* W_aud, h3_bf16* patches, float* x_out, float* pos_out, uint8_t* mod_out,
                  void* stream);

/* A3 / A8.  xm = LayerNorm(x) * (1 + scale_m) + shift_m, m = modality of the
 * row's range, branch H3_MSA or H3_MLP selects the (shift, scale) pair
 * ([shouss] §3, §3.1).  LayerNorm without affine, biased variance, eps_ln.
 *   x [L_pad][D] fp32 -> xm [L_pad][D] bf16 (padding rows written as 0). */
int h3_adaln_norm_modulate(const h3_dims* dims, const h3_ranges* ranges, const float* x, const float* mod,
                           int branch, h3_bf16* xm, void* stream);

/* A4 + A5.  [q | k | v] = xm * Wqkv^T (Wqkv [3I][D]); with
 * H3_QK_NORM_ROPE_IN_QKV, every 128-wide head of q and k is RMS-normalised
 * (eps_qk) and scaled by qn_w / kn_w [128], then rotated by the 3-D RoPE:
 * head_dim splits into t | h | w sections (rope_t, rope_h, rope_w); pair
 * (2i, 2i+1) of a section of width d turns by pos_axis * theta^(-2i/d)
 * ([shouss] §3.2: per-head RMSNorm then positional encoding; [gojay] §7.4).
 * Without the flag q and k are written as the GEMM leaves them (rounded to
 * bf16) and qn_w, kn_w, pos are not read (they may be NULL).
 *   pos [L_pad][3] fp32;  q, k, v out: head-major [H][L_pad][128] bf16. */
int h3_qkv_qknorm_mrope(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* xm, const h3_bf16* Wqkv,
                        const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags, h3_bf16* q,
                        h3_bf16* k, h3_bf16* v, void* stream);

/* A6.  o = softmax(q k^T / sqrt(128)) v per head over all L valid tokens,
 * non-causal; keys >= L are masked ([shouss] §5).  q, k, v: head-major
 * [H][L_pad][128] bf16 as written by h3_qkv_qknorm_mrope with the same
 * H3_QK_NORM_ROPE_IN_QKV setting.
 * Without H3_QK_NORM_ROPE_IN_QKV: q, k are raw; qn_w, kn_w and pos
 * [L_pad][3] fp32 are required, and the split-softmax kernel normalises and
 * rotates them in its prologue (four extra warps, one row each) before
 * taking the same bounded softmax as below.  Nothing recomputes a CTA whose
 * bound fails there: it leaves NaN in its first output element and
 * h3_device_status then returns H3_ERR_BOUND (code 2).  The bound holds by
 * construction for max|qn_w| * max|kn_w| <= 3.6.
 * With the flag, pos is unused and may be NULL:
 *   qn_w, kn_w: the norm weights q and k were normalised with, or both NULL.
 *     Given (bf16 q, k), the softmax needs no running maximum: every score
 *     lies within sqrt(128) max|qn_w| max|kn_w| of 0, so the exponentials are
 *     taken against that bound, each row's over two warps.  A CTA whose
 *     scores break the bound (q, k not normalised as stated) or whose bound
 *     is too wide for fp32 (scores past +-60 in log2 units) is recomputed by
 *     the general kernel in a second launch: the result is the same either
 *     way.  NULL: the general kernel (moving softmax reference) alone.
 * With flags & H3_QK_E4M3, q and k are the e4m3 codes written by
 * h3_qkv_qknorm_mrope_e4m3 with that flag (one byte per element) and qn_w,
 * kn_w are required: the code scales follow from them.
 *   o [L_pad][H*128] bf16, token-major; rows >= L written as 0. */
int h3_attention(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* q, const h3_bf16* k,
                 const h3_bf16* v, const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags,
                 h3_bf16* o, void* stream);

/* A7.  x[r] += gate_m[branch] (.) (o * Wo^T)[r] for valid rows r, m = modality
 * of r ([shouss] §3: shared attention + modality gate + residual).
 *   x [L_pad][D] fp32 in/out; o [L_pad][I] bf16; Wo [D][I] bf16. */
int h3_gated_residual(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* o,
                      const h3_bf16* Wo, const float* mod, int branch, void* stream);

/* Bytes of the h3_ffn_swiglu workspace: L_pad * F * sizeof(bf16). */
size_t h3_ffn_workspace_bytes(const h3_dims* dims, int L_pad);

/* A9.  h = SiLU(xm Wg^T) (.) (xm Wu^T) into ws, then
 * x[r] += gate_mlp_m (.) (h Wd^T)[r] ([shouss] §3, §3.2).
 *   Wgu [2F][D] bf16 = [gate rows; up rows]; Wd [D][F] bf16;
 *   ws  caller-owned scratch of h3_ffn_workspace_bytes() bytes. */
int h3_ffn_swiglu(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* xm,
                  const h3_bf16* Wgu, const h3_bf16* Wd, const float* mod, h3_bf16* ws, void* stream);

/* Size in bytes of the device array that h3_ffn_swiglu_noalloc uses as its
 * workspace: 32 MiB, i.e. L_pad * F <= 16 Mi elements (at F = 14336, up to
 * L_pad = 1152 tokens). */
#define H3_FFN_STATIC_WS_BYTES (32u * 1024u * 1024u)

/* h3_ffn_swiglu without a caller workspace; nothing is allocated.  No
 * counterpart on the pages: this entry point exists for callers that own
 * only their inputs and outputs and cannot obtain device memory for scratch
 * (an operator or plugin interface that passes tensors but no workspace, a
 * process whose device memory is all reserved by another allocator, a
 * serving loop that must not allocate on its hot path).  Same arguments and
 * result as h3_ffn_swiglu minus ws.
 *   - The workspace is a fixed device array of H3_FFN_STATIC_WS_BYTES inside
 *     the library, present on every GPU that loads it until the process
 *     exits.  Calls with L_pad * F * 2 > H3_FFN_STATIC_WS_BYTES are rejected
 *     with H3_ERR_SHAPE before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     calls whose kernels overlap on the GPU (other streams, other host
 *     threads) race on it and must be serialised by the caller.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
int h3_ffn_swiglu_noalloc(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* xm,
                          const h3_bf16* Wgu, const h3_bf16* Wd, const float* mod, void* stream);

/* A10 (a reading: the pages say only that the output layers are
 * modality-specific, [gojay] §5).  Non-affine LayerNorm of x into hn, then
 * v_video = unpatchify(hn_video * W_vhead^T) [T][Hl][Wl][C_lat] fp32 and
 * v_audio = hn_audio * W_ahead^T [audio_channels][n_audio][C_audio] fp32.
 *   W_vhead [4*C_lat][D], W_ahead [C_audio][D] bf16; hn [L_pad][D] bf16 scratch. */
int h3_head_unpack(const h3_dims* dims, const h3_ranges* ranges, const float* x, const h3_bf16* W_vhead,
                   const h3_bf16* W_ahead, int T, int Hl, int Wl, int C_lat, int audio_channels, int n_audio,
                   int C_audio, h3_bf16* hn, float* v_video, float* v_audio, void* stream);

/* A10 + A11 fused: the head of h3_head_unpack with the Euler step of each
 * latent in its GEMM epilogues, so the velocities are never written out:
 *   lat_video += (sigma_video_next - sigma_video) * v_video,
 *   lat_audio += (sigma_audio_next - sigma_audio) * v_audio,
 * with v_video, v_audio as h3_head_unpack computes them (same accumulation;
 * the update is the same fused multiply-add as h3_euler_step, so the result
 * equals h3_head_unpack followed by h3_euler_step on each latent bit for
 * bit).  Each modality has its own sigmas (its own shifted schedule,
 * [shouss] §6); text rows are not touched ([shouss] §5).  lat_video
 * [T][Hl][Wl][C_lat] and lat_audio [audio_channels][n_audio][C_audio] are
 * fp32 device arrays updated in place; lat_video_bf16 / lat_audio_bf16, when
 * not NULL, receive the updated latents rounded to bf16 (the next step's
 * transformer input), same layouts.  hn [L_pad][D] bf16 scratch.  Errors as
 * h3_head_unpack. */
int h3_head_euler(const h3_dims* dims, const h3_ranges* ranges, const float* x, const h3_bf16* W_vhead,
                  const h3_bf16* W_ahead, int T, int Hl, int Wl, int C_lat, int audio_channels, int n_audio,
                  int C_audio, h3_bf16* hn, float* lat_video, float* lat_audio, float sigma_video,
                  float sigma_video_next, float sigma_audio, float sigma_audio_next, h3_bf16* lat_video_bf16,
                  h3_bf16* lat_audio_bf16, void* stream);

/* NEXT-3 (a reading, G22): the AdaLN modulation producer of one block.
 * The pages put ~13B parameters in the AdaLN branch and say its outputs
 * depend only on the timestep and the condition, so they can be computed
 * ahead and cached ([gojay] §5; [shouss] §3.1: 6D features per modality,
 * 18D in all).  Read here as one linear per block on SiLU of a conditioning
 * vector (timestep + condition embedding, computed by the caller; its width
 * D/2 reproduces the 13B count at 50 blocks), no bias:
 *   mod[i] = W * SiLU(c[i]), viewed as [3][6][D] (layout of mod elsewhere).
 *   c   [n][c_dim] fp32 device (n >= 1 vectors, e.g. one per sampler step)
 *   W   [18 D][c_dim] bf16 device, c_dim a multiple of 8
 *   ws  scratch of h3_adaln_workspace_bytes(n, c_dim) bytes (SiLU(c) in bf16)
 *   mod [n][3][6][D] fp32 device output, rows ld_mod floats apart (0: 18 D;
 *       e.g. n_blocks * 18 D to fill block b's column of a
 *       [step][block][3][6][D] cache, mod pointing at block b)
 * SiLU(c) enters the tensor-core GEMM as bf16 (fp32 accumulation).
 * Errors: H3_ERR_SHAPE (n <= 0), H3_ERR_UNSUPPORTED (c_dim), NULL / alignment
 * as elsewhere; nothing is launched on error. */
size_t h3_adaln_workspace_bytes(int n, int c_dim);
int h3_adaln_modulation(const h3_dims* dims, const float* c, int n, int c_dim, const h3_bf16* W, h3_bf16* ws,
                        float* mod, int64_t ld_mod, void* stream);

/* A11.  lat[i] += (sigma_next - sigma) * vel[i] for i < n: one Euler step of
 * the rectified-flow ODE on a generation target (x0 = x - sigma v;
 * [shouss] §5, §6).  lat, vel: fp32 device arrays of n elements. */
int h3_euler_step(float* lat, const float* vel, int64_t n, float sigma, float sigma_next, void* stream);

/* Block weights and scratch buffers for h3_block_forward (all device
 * pointers, layouts as in the individual calls). */
typedef struct h3_block_weights {
  const h3_bf16* Wqkv; /* [3I][D] */
  const h3_bf16* qn_w; /* [128] */
  const h3_bf16* kn_w; /* [128] */
  const h3_bf16* Wo;   /* [D][I] */
  const h3_bf16* Wgu;  /* [2F][D], gate rows then up rows */
  const h3_bf16* Wd;   /* [D][F] */
} h3_block_weights;

typedef struct h3_block_buffers {
  h3_bf16* xm;         /* [L_pad][D] */
  h3_bf16* q;          /* [H][L_pad][128] */
  h3_bf16* k;          /* [H][L_pad][128] */
  h3_bf16* v;          /* [H][L_pad][128] */
  h3_bf16* o;          /* [L_pad][I] */
  h3_bf16* ws;         /* h3_ffn_workspace_bytes() */
} h3_block_buffers;

/* One whole block on x in place: h3_adaln_norm_modulate (MSA),
 * h3_qkv_qknorm_mrope, h3_attention, h3_gated_residual, h3_adaln_norm_modulate
 * (MLP), h3_ffn_swiglu, in the order of [shouss] §3 (norm + modality
 * shift/scale -> shared attention + gate + residual -> norm + shift/scale ->
 * shared gated FFN + gate + residual).  Same arguments and errors as those
 * calls; nothing is launched if any argument is invalid.  flags: 0 or
 * H3_QK_NORM_ROPE_IN_QKV, passed to the QKV and attention calls (where the
 * Q/K norm and RoPE run). */
int h3_block_forward(const h3_dims* dims, const h3_ranges* ranges, float* x, const float* mod, const float* pos,
                     const h3_block_weights* w, const h3_block_buffers* buf, int flags, void* stream);

/* NEXT-3, a reading: the text refiner ("MiniMax-H3: native joint audio-video
 * generation" (note.shouss.top) §3.2 config table: 2 text refiner blocks that
 * prepare the text before the trunk; their structure is not stated).  Here
 * a refiner block has the trunk block's form (h3_block_forward) and runs over
 * the text range alone: the packed rows [0, count[TEXT]) of x (text comes
 * first in the packing) as a text-only sequence, in place, each block with
 * its own weights w[b] and modulation mods[b] ([3][6][D], only the text slot
 * read); audio and video rows of x are read by nothing and left unchanged.
 * pos: the packed positions (text rows are at (0, 0, 0)); buf: buffers for
 * h3_block_forward at the packed L_pad (the text-only pass uses less).  No-op
 * when there is no text or n_blocks == 0. */
int h3_text_refine(const h3_dims* dims, const h3_ranges* ranges, float* x, int n_blocks, const float* const* mods,
                   const float* pos, const h3_block_weights* w, const h3_block_buffers* buf, int flags, void* stream);

/* A11 for a sampler loop: h3_euler_step, and also writes the updated latent
 * rounded to bf16 into lat_bf16 (the transformer input of the next step). */
int h3_euler_step_bf16(float* lat, const float* vel, int64_t n, float sigma, float sigma_next, h3_bf16* lat_bf16,
                       void* stream);

/* Diagnostic for failure detection: one device thread waits, with the given
 * limit (nanoseconds, at most 10 s), on an mbarrier that nothing arrives on.
 * The wait gives up and records code 1 in the device error word exactly as a
 * stalled pipeline wait would; h3_device_status then returns H3_ERR_TIMEOUT.
 * Nothing faults and the context stays usable. */
int h3_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Synchronise `stream`, then report (and clear) the device error word that
 * bounded device-side waits set when they give up.  *code_out = 0 when no
 * wait failed.  Returns H3_ERR_TIMEOUT if one did, H3_ERR_CUDA on a CUDA
 * error, else H3_OK. */
int h3_device_status(void* stream, int* code_out);

/* Set the time limit (nanoseconds, > 0) of every device-side wait for
 * kernels launched afterwards on the current device (default 2 s). */
int h3_set_wait_limit_ns(uint64_t ns);

/* ------------------------------------------------------------------------
 * FP8 (e4m3) GEMMs.  The pages report community FP8 / INT4 quantisations of
 * the trunk ("H3's omni-modal ambition" (0539edu.com), ecosystem paragraph)
 * and fix no format; these entry points take the block's four GEMMs to e4m3
 * tensor-core MMAs (tcgen05 kind::f8f6f4, fp32 accumulate) with this scheme:
 *   - e4m3 is the OCP OFP8 E4M3 format (bias 7, 3 mantissa bits, largest
 *     finite 448, no infinities); encoding rounds to nearest, ties to even,
 *     saturating to +-448, sign bit kept (h3_e4m3 holds one code).
 *   - Row scaling: amax = max |row|; rscale = 448 / amax and scale =
 *     amax / 448 (IEEE fp32 divisions); code = e4m3(row * rscale) with the
 *     product rounded to fp32; a zero row has scale 0 and codes 0.
 *   - Activations carry one scale per token (row), weights one per output
 *     channel (row of the [out][in] weight).  A GEMM then computes
 *     acc[m][n] * a_scale[m] * b_scale[n] and applies the same fused
 *     epilogue as its bf16 counterpart.
 * Attention stays bf16 unless H3_QK_E4M3 is set: then q and k cross from
 * the QKV call to attention as e4m3 codes with one static scale each,
 *   s_q = fp32(sqrt(128) * max|qn_w|) / 448 (fp32 arithmetic, sqrt(128) as
 *   the fp32 constant 11.3137085), code = e4m3(fp32(q * fp32(1 / s_q)))
 * written as 448 / fp32(11.3137085 * max|qn_w|), and likewise for k with
 * kn_w.  RMSNorm then RoPE bound every element of a head row by
 * sqrt(128) max|w|, so no code saturates; S = s_q s_k (Q8 K8^T).
 * Code matrices are row-major bytes; every row length is a multiple of 16
 * bytes as for the bf16 calls (D % 64, I, F % 128). */
typedef uint8_t h3_e4m3;

/* Row quantisation of a bf16 matrix (weights offline; activations between
 * calls).  in [rows][cols] with row stride ld_in elements -> q [rows][cols]
 * codes with row stride ld_q bytes, scale [rows] fp32.  cols, ld_in and ld_q
 * must be multiples of 8 and in, q 16-byte aligned. */
int h3_quantize_rows_e4m3(const h3_bf16* in, int64_t ld_in, int rows, int cols, h3_e4m3* q, int64_t ld_q,
                          float* scale, void* stream);

/* A3 / A8 with e4m3 output: the fp32 values h3_adaln_norm_modulate would
 * round to bf16 are row-quantised instead.  xq [L_pad][D] codes, xs [L_pad]
 * fp32 (padding rows: codes 0, scale 0). */
int h3_adaln_norm_modulate_e4m3(const h3_dims* dims, const h3_ranges* ranges, const float* x, const float* mod,
                                int branch, h3_e4m3* xq, float* xs, void* stream);

/* A4 + A5 from e4m3 operands: as h3_qkv_qknorm_mrope with xm = (xq, xs)
 * [L_pad][D] and Wqkv = (Wq, Ws) [3I][D], Ws per output channel.  q, k, v
 * bf16 head-major [H][L_pad][128]; with flags & H3_QK_E4M3, q and k receive
 * e4m3 codes instead, [H][L_pad][128] bytes (the buffers may be the bf16
 * ones: half of each is used), v stays bf16. */
int h3_qkv_qknorm_mrope_e4m3(const h3_dims* dims, const h3_ranges* ranges, const h3_e4m3* xq, const float* xs,
                             const h3_e4m3* Wq, const float* Ws, const h3_bf16* qn_w, const h3_bf16* kn_w,
                             const float* pos, int flags, h3_bf16* q, h3_bf16* k, h3_bf16* v, void* stream);

/* A7 from e4m3 operands: as h3_gated_residual with o = (oq, os) [L_pad][I]
 * (e.g. the attention output through h3_quantize_rows_e4m3) and
 * Wo = (Wq, Ws) [D][I]. */
int h3_gated_residual_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_e4m3* oq,
                           const float* os, const h3_e4m3* Wq, const float* Ws, const float* mod, int branch,
                           void* stream);

/* Bytes of the h3_ffn_swiglu_e4m3 workspace: the bf16 hidden state
 * [L_pad][F], its codes [L_pad][F] and their scales [L_pad] fp32. */
size_t h3_ffn_e4m3_workspace_bytes(const h3_dims* dims, int L_pad);

/* A9 from e4m3 operands: h = bf16(SiLU(xm Wg^T) (.) (xm Wu^T)) with
 * xm = (xq, xs) and Wgu = (Wgu_q, Wgu_s) [2F][D] (gate rows then up rows),
 * then h row-quantised, then x[r] += gate_mlp_m (.) (h Wd^T)[r] with
 * Wd = (Wd_q, Wd_s) [D][F].  ws: caller-owned scratch of
 * h3_ffn_e4m3_workspace_bytes() bytes, 256-byte aligned. */
int h3_ffn_swiglu_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_e4m3* xq,
                       const float* xs, const h3_e4m3* Wgu_q, const float* Wgu_s, const h3_e4m3* Wd_q,
                       const float* Wd_s, const float* mod, void* ws, void* stream);

/* Block weights (e4m3 codes with per-output-channel scales) and buffers for
 * h3_block_forward_e4m3. */
typedef struct h3_block_weights_e4m3 {
  const h3_e4m3* Wqkv; const float* Wqkv_s; /* [3I][D], [3I] */
  const h3_bf16* qn_w;                      /* [128] */
  const h3_bf16* kn_w;                      /* [128] */
  const h3_e4m3* Wo;   const float* Wo_s;   /* [D][I], [D] */
  const h3_e4m3* Wgu;  const float* Wgu_s;  /* [2F][D], [2F] */
  const h3_e4m3* Wd;   const float* Wd_s;   /* [D][F], [D] */
} h3_block_weights_e4m3;

typedef struct h3_block_buffers_e4m3 {
  h3_e4m3* xq; float* xs; /* [L_pad][D], [L_pad] */
  h3_bf16* q;             /* [H][L_pad][128] */
  h3_bf16* k;
  h3_bf16* v;
  h3_bf16* o;             /* [L_pad][I] */
  h3_e4m3* oq; float* os; /* [L_pad][I], [L_pad] */
  void* ws;               /* h3_ffn_e4m3_workspace_bytes() */
} h3_block_buffers_e4m3;

/* One whole block with e4m3 GEMMs: h3_adaln_norm_modulate_e4m3 (MSA),
 * h3_qkv_qknorm_mrope_e4m3, h3_attention (bf16, or e4m3 Q K^T with
 * flags & H3_QK_E4M3: buf->q, buf->k then hold codes), h3_quantize_rows_e4m3
 * of o, h3_gated_residual_e4m3, h3_adaln_norm_modulate_e4m3 (MLP),
 * h3_ffn_swiglu_e4m3.  Nothing is launched if any argument is invalid. */
int h3_block_forward_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const float* mod,
                          const float* pos, const h3_block_weights_e4m3* w, const h3_block_buffers_e4m3* buf,
                          int flags, void* stream);

/* ------------------------------------------------------------------------
 * Sequence parallelism (Ulysses), the pages' own multi-GPU deployment of the
 * trunk ([gojay] §7.2: Ulysses degree 4).  N ranks (N <= H3_SP_MAX_RANKS,
 * H % N == 0) each hold a contiguous shard of L_shard rows of the packed
 * sequence: rank r owns global rows [r L_shard, (r + 1) L_shard) of a
 * sequence padded to L_total = N L_shard.  Everything token-local (LN +
 * modulation, the GEMMs, the FFN, the residual) runs on the shard with the
 * shard's h3_ranges.  Attention needs every token of a head, so the QKV
 * call writes head group g (heads [g H/N, (g + 1) H/N)) of its shard
 * straight into rank g's q/k/v buffers (an all-to-all fused into the GEMM
 * epilogue), and the attention call writes each output row straight into
 * the o buffer of the row's owner (the second all-to-all, fused into the
 * attention epilogue).  Peer buffers are device pointers the caller maps
 * (CUDA IPC or symmetric memory between GPUs; plain local buffers when the
 * ranks share one GPU).  Between the QKV calls of all ranks and any
 * attention call, and between the attention calls and the out-projections,
 * every rank's writes must be complete and visible: the caller orders them
 * (a barrier on the streams, e.g. a collective or event wait). */
#define H3_SP_MAX_RANKS 8

typedef struct h3_sp_layout {
  int n_ranks;   /* N */
  int rank;      /* this rank */
  int L;         /* valid tokens of the whole sequence */
  int L_shard;   /* rows per shard, a multiple of 128: ceil(L / N / 128) * 128 */
  int L_total;   /* N * L_shard */
  int row0;      /* rank * L_shard: first global row of this shard */
  int heads;     /* H / N: heads per rank after the exchange */
} h3_sp_layout;

/* Host only.  The layout of rank `rank` of n_ranks for the global ranges,
 * and the shard's own ranges (modality ranges intersected with the shard,
 * relative to its first row; shard->L = its valid rows, shard->L_pad =
 * L_shard).  Every shard must hold at least one valid row:
 * L > (n_ranks - 1) * L_shard, else H3_ERR_SHAPE. */
int h3_sp_make_layout(const h3_dims* dims, const h3_ranges* global, int n_ranks, int rank, h3_sp_layout* out,
                      h3_ranges* shard);

/* Device pointers of every rank's exchange buffers (index = rank):
 *   q[g], k[g], v[g]: rank g's [H/N][L_total][128] bf16 (head-major; global
 *                     row order, so the attention of rank g sees the whole
 *                     sequence for its heads); with H3_QK_E4M3, q[g] and
 *                     k[g] hold one-byte e4m3 codes in the same layout
 *   o[g]:             rank g's [L_shard][H * 128] bf16 attention output */
typedef struct h3_sp_peers {
  h3_bf16* q[H3_SP_MAX_RANKS];
  h3_bf16* k[H3_SP_MAX_RANKS];
  h3_bf16* v[H3_SP_MAX_RANKS];
  h3_bf16* o[H3_SP_MAX_RANKS];
} h3_sp_peers;

/* A4 + A5 on this rank's shard (xm [L_shard][D], pos [L_shard][3]) with the
 * q, k, v of head h written to rank h / (H/N), local head h % (H/N), global
 * row row0 + m: the QKV GEMM and the first all-to-all in one kernel. */
int h3_qkv_qknorm_mrope_sp(const h3_dims* dims, const h3_ranges* shard, const h3_sp_layout* layout,
                           const h3_bf16* xm, const h3_bf16* Wqkv, const h3_bf16* qn_w, const h3_bf16* kn_w,
                           const float* pos, int flags, const h3_sp_peers* peers, void* stream);

/* NEXT-1 with NEXT-2: h3_qkv_qknorm_mrope_sp on e4m3 operands (xq [L_shard][D]
 * codes with per-row scales xs, Wq [3I][D] codes with per-output-channel
 * scales Ws, as h3_qkv_qknorm_mrope_e4m3).  With flags & H3_QK_E4M3 the q, k
 * that cross to the head-group ranks are e4m3 codes (half the bytes of
 * bf16; scales from qn_w, kn_w), and every rank's h3_attention_sp then takes
 * the same flag. */
int h3_qkv_qknorm_mrope_sp_e4m3(const h3_dims* dims, const h3_ranges* shard, const h3_sp_layout* layout,
                                const h3_e4m3* xq, const float* xs, const h3_e4m3* Wq, const float* Ws,
                                const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags,
                                const h3_sp_peers* peers, void* stream);

/* A6 for this rank's H/N heads over all L tokens (its q, k, v =
 * peers->q/k/v[rank], filled by every rank's h3_qkv_qknorm_mrope_sp), with
 * output row R (global) written to peers->o[R / L_shard], row R % L_shard,
 * columns of head (rank H/N + h): attention and the second all-to-all in
 * one kernel.  Rows >= L are written as 0.  qn_w, kn_w: as for
 * h3_attention (the norm weights q and k were normalised with, selecting
 * the split-softmax kernel, or both NULL; required with H3_QK_E4M3, where q
 * and k are e4m3 codes). */
int h3_attention_sp(const h3_dims* dims, const h3_sp_layout* layout, const h3_sp_peers* peers,
                    const h3_bf16* qn_w, const h3_bf16* kn_w, int flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* H3_H */
