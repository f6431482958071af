// Internal launch interfaces shared by the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace h3 {

typedef __nv_bfloat16 bf16;

// Epilogue variants of the tensor-core GEMM (out = A[M,K] * B[N,K]^T).
enum EpiMode : int {
  EPI_STORE_F32 = 0,    // out_f32[(row_off + m) * ldo + n] = acc
  EPI_GATED_RESID = 1,  // x[(row_off + m) * ldo + n] += gate[mod(row)][n] * acc
  EPI_SWIGLU = 2,       // ws[m * ldo + n] = bf16(SiLU(acc_gate) * acc_up)
  EPI_QKV = 3,          // per-head Q/K RMSNorm + 3-D RoPE, head-major bf16 scatter
  EPI_UNPATCH = 4,      // video head: acc row -> latent gather (inverse patchify), f32
};

struct GemmEpilogue {
  int mode;
  int M, N;          // valid output rows / columns of this GEMM
  int row_off;       // packed-sequence row of GEMM row 0
  long ldo;          // output row stride (elements)
  void* out;         // EPI_STORE_F32 / EPI_GATED_RESID (x) / EPI_SWIGLU (ws) / EPI_UNPATCH
  // modality ranges (packed rows) for gate selection
  int rstart[3], rcount[3];
  const float* mod;  // [3][6][D] fp32
  int gate_slot;     // 2 (gate_msa) or 5 (gate_mlp)
  int D;
  // EPI_QKV
  bf16* q;
  bf16* k;
  bf16* v;
  const bf16* qn_w;
  const bf16* kn_w;
  const float* pos;  // [L_pad][3]
  int L_pad, I;
  int rope_t, rope_h, rope_w;
  float theta, eps_qk;
  // EPI_QKV with qk_e4m3: q and k are written as e4m3 codes (q, k then point
  // to [H][L_pad][128] bytes) of value * 448 / (sqrt(128) max|w|), w the
  // head's norm weight; v stays bf16
  int qk_e4m3;
  // EPI_QKV with qk_raw: q and k are written as they leave the GEMM (no
  // RMSNorm, no RoPE), for attention to take both in its prologue
  int qk_raw;
  // EPI_UNPATCH: token grid (T, Ht, Wt), latent channels
  int Ht, Wt, C_lat;
  // EPI_STORE_F32 / EPI_UNPATCH with euler != 0: out holds a latent that
  // takes one Euler step in place, out[i] = out[i] + dsigma * acc (acc is the
  // velocity), and out_bf16 (when set, same layout) receives bf16(out[i])
  // after the update
  int euler;
  float dsigma;
  bf16* out_bf16;
  // e4m3 operands: acc[m][n] *= a_scale[m] * b_scale[n] before the epilogue
  // (a_scale per A row, b_scale per B row); null for bf16 operands.  Set by
  // launch_gemm from GemmProblem.
  const float* a_scale;
  const float* b_scale;
  int a_rows, b_rows;
  // EPI_QKV, sequence parallel (sp_n > 0): head h of GEMM row m goes to rank
  // h / sp_heads, local head h % sp_heads, row sp_row0 + m of its
  // [sp_heads][sp_L_total][128] buffers sp_q / sp_k / sp_v.
  int sp_n, sp_heads, sp_L_total, sp_row0;
  bf16* sp_q[8];
  bf16* sp_k[8];
  bf16* sp_v[8];
};

struct GemmProblem {
  const void* A;  // bf16 [M, K] row-major
  long lda;       // elements
  const void* B;  // bf16 [N_b, K] row-major ([out, in] weight)
  long ldb;
  int N_b_rows;   // rows of B (for the tensor map extent)
  int M, K;
  int n_tiles;    // number of 256-wide (or 128-pair for SwiGLU) column tiles
  int group_m;    // tile order: bands of group_m row tiles sweep all column tiles (L2 reuse of A)
  int pair;       // 1: CTA-pair kernel (256 x 256 tiles over two SMs) when M > 128; 0: one CTA per tile
  int b_second_half_off;  // SwiGLU: row offset of the "up" half in B (= F); else 128
  // e4m3 operands (kind::f8f6f4): A and B hold one-byte codes (lda / ldb in
  // bytes), scaled per A row and per B row; 0 for bf16.
  int f8;
  const float* a_scale;
  const float* b_scale;
  GemmEpilogue epi;
};

// Launch one tensor-core GEMM on `stream`.  Returns a cudaError_t.
cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream);

// Attention over head-major q, k, v [H][L_pad][128] -> o [L_pad][H*128].
struct AttnProblem {
  const bf16* q;
  const bf16* k;
  const bf16* v;
  bf16* o;
  int H, L, L_pad;
  float scale_log2;  // log2(e) / sqrt(head_dim)
  // Sequence parallel (sp_n > 0): o row R goes to sp_o[R / sp_L_shard], row
  // R % sp_L_shard, row stride sp_ld elements, head column offset
  // (sp_head0 + h) * 128; o is unused.
  int sp_n, sp_L_shard, sp_head0;
  long sp_ld;
  bf16* sp_o[8];
  // qk8: q, k hold e4m3 codes (one byte per element) written by the QKV
  // epilogue with qk_e4m3; qn_w, kn_w give their scales
  int qk8;
  const bf16* qn_w;
  const bf16* kn_w;
  // prologue != 0: q, k are raw (the QKV GEMM without its norm and RoPE),
  // and attention applies the per-head RMSNorm (weights qn_w, kn_w, eps) and
  // the 3-D RoPE (positions pos [L_pad][3], sections rope_t | rope_h |
  // rope_w, base theta) in its prologue
  int prologue;
  const float* pos;
  int rope_t, rope_h, rope_w;
  float theta, eps_qk;
};
cudaError_t launch_attention(const AttnProblem& p, cudaStream_t stream);

// Memory-bound kernels.
cudaError_t launch_pack(const bf16* video, int T, int Hl, int Wl, int C_lat, int n_audio, int audio_channels,
                        const int* rstart, const int* rcount, int L, int L_pad, bf16* patches, float* pos,
                        uint8_t* mod_ids, float* x, int D, cudaStream_t stream);
cudaError_t launch_ln_modulate(const float* x, const float* mod, int branch, const int* rstart, const int* rcount,
                               int L, int L_pad, int D, float eps, bf16* out, cudaStream_t stream);
cudaError_t launch_ln_modulate_e4m3(const float* x, const float* mod, int branch, const int* rstart,
                                    const int* rcount, int L, int L_pad, int D, float eps, uint8_t* out,
                                    float* out_scale, cudaStream_t stream);
cudaError_t launch_quantize_rows_e4m3(const bf16* in, long ld_in, int rows, int cols, uint8_t* q, long ld_q,
                                      float* scale, cudaStream_t stream);
cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_euler_bf16(float* lat, const float* vel, long long n, float dsigma, bf16* out,
                              cudaStream_t stream);
cudaError_t launch_euler(float* lat, const float* vel, long long n, float dsigma, cudaStream_t stream);
cudaError_t launch_silu_bf16(const float* c, long long n, bf16* a, cudaStream_t stream);

int num_sms();

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) once per
// device (function attributes are per device context).
cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned long long* done_mask);

}  // namespace h3
