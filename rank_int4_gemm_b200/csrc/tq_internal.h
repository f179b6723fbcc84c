// tq_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace tq {

// Host-side knobs for experiments (0 = automatic choice).
struct Tuning {
  int split_k = 0;        // decode GEMM: number of K splits
  int pdl = 1;            // launch the GEMM with programmatic dependent launch
  int layer_a8 = 1;       // tq_w4a4_lr_layer at M > 128: codes one per byte
};
Tuning& tuning();

// `signs`: n_rht randomized Hadamard sign masks [n_rht][K / 32] (rotation
// by D_1 H ... D_n H, composed transforms), or null for the plain Hadamard.
cudaError_t launch_pack_weight(const float* Rt, int N, int K, int had_block, uint8_t* Wq,
                               float* s_w, cudaStream_t stream, const uint32_t* signs = nullptr,
                               int n_rht = 1);

cudaError_t launch_quantize_act(const uint16_t* X, int M, int K, int had_block,
                                const uint16_t* L1t, int r, uint8_t* Xq, float* s_x,
                                float* XL1, cudaStream_t stream, const uint32_t* signs = nullptr,
                                int n_rht = 1);

// The butterfly activation kernel writing one code per byte and bf16(X L1)
// (the int8-code GEMM's operands), with an optional sign mask.
cudaError_t launch_quantize_act_bf_i8(const uint16_t* X, int M, int K, int had_block,
                                      const uint16_t* L1t, int r, int8_t* Xq8, float* s_x,
                                      uint16_t* XL1b, cudaStream_t stream,
                                      const uint32_t* signs = nullptr, int n_rht = 1);

// Activation stage on tensor cores (many tokens): rotation and X L1 as MMAs.
// Codes packed (Xq, [M][K/2]) or one int8 per code (Xq8, [M][K]); X L1 as
// fp32 (XL1) and / or rounded to bf16 (XL1b), either may be null.
bool act_tc_supported(int M, int K, int had_block, int r);
// z_x non-null: asymmetric codes (zero-point = row minimum, codes 0..15
// stored as code - 8), s_x = range / 15.  signs non-null: one randomized
// Hadamard mask ([K / 32] words), codes of x D H (symmetric only).
cudaError_t launch_act_tc(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t,
                          int r, uint8_t* Xq, int8_t* Xq8, float* s_x, float* XL1, uint16_t* XL1b,
                          cudaStream_t stream, float* z_x = nullptr,
                          const uint32_t* signs = nullptr);

// GEMM with one int8 per activation code (weights expanded into TMEM).
struct GemmA8Args {
  const int8_t* Xq8;      // [M][K]
  const float* s_x;
  const uint8_t* Wq;      // [N][K/2]
  const float* s_w;
  const uint16_t* XL1b;   // [M][r] bf16
  const uint16_t* L2t;    // [N][r] bf16
  int M, N, K, r;
  uint16_t* Y;            // [M][N], or [M][N/2] with swiglu
  void* ws;               // status word at offset 0
  int swiglu = 0;         // rows alternate gate / up: Y = silu(gate) * up
  const float* z_x = nullptr;     // asymmetric activation codes: [M] zero-points
  const int32_t* wsum = nullptr;  //   and [N] weight code sums
  const float* s_xl1 = nullptr;   // INT4 low-rank branch: [M] and [N] scales (XL1b and
  const float* s_l2 = nullptr;    //   L2t then hold integer codes in bf16)
  void* sk = nullptr;             // stream-K scratch (gemm_a8_sk_bytes(), zero-filled before
                                  //   first use), or null for tile-by-tile CTAs only
};
cudaError_t launch_gemm_a8(const GemmA8Args& a, cudaStream_t stream);
// Bytes of the a8 GEMM's stream-K scratch: ready flags and INT32 partial
// tiles for up to one split tile per CTA.
size_t gemm_a8_sk_bytes();
cudaError_t launch_pack_lowrank_q4(const uint16_t* L1t, const uint16_t* L2t, int N, int K, int r,
                                   int had_block, int8_t* qL1, float* s_L1, uint16_t* qL2,
                                   float* s_L2, cudaStream_t stream);
// X L1 of the INT4 low-rank branch from the activation codes (tq_qlr.cu):
// INT32 on the tensor cores, requantized per token; acc [M][r] INT32 is
// scratch for ranks above 256, status the timeout word.
cudaError_t launch_xl1_codes(const int8_t* Xq8, const int8_t* qL1, const float* s_x,
                             const float* s_L1, int M, int K, int r, uint16_t* XL1q, float* s_xl1,
                             int32_t* acc, uint32_t* status, cudaStream_t stream);
cudaError_t launch_requant_xl1(const int32_t* acc, const float* s_x, const float* s_L1, int M,
                               int r, uint16_t* XL1q, float* s_xl1, cudaStream_t stream);
cudaError_t launch_weight_code_sums(const uint8_t* Wq, int N, int K, int32_t* wsum,
                                     cudaStream_t stream);
cudaError_t launch_pack_gate_up(const uint8_t* Wq_g, const float* s_w_g, const uint16_t* L1t_g,
                                const uint16_t* L2t_g, const uint8_t* Wq_u, const float* s_w_u,
                                const uint16_t* L1t_u, const uint16_t* L2t_u, int N, int K, int r,
                                uint8_t* Wq2, float* s_w2, uint16_t* L1t2, uint16_t* L2t2,
                                cudaStream_t stream);

struct GemmArgs {
  const uint8_t* Xq;
  const float* s_x;
  const uint8_t* Wq;
  const float* s_w;
  const float* XL1;
  const uint16_t* L2t;
  int M, N, K, r;
  uint16_t* Y;          // bf16 output (null in accumulator-debug mode)
  int32_t* acc_out;     // raw INT32 accumulators (debug mode), or null
  void* ws;
  size_t ws_bytes;
};

size_t gemm_workspace_bytes(int M, int N, int K, int r);
// Status of the GEMM's operand arguments (null pointers, shape limits,
// alignment), without the workspace and device checks; TQ_OK when valid.
int gemm_operand_status(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w,
                        const float* XL1, const uint16_t* L2t, int M, int N, int K, int r,
                        const uint16_t* Y, const int32_t* acc);
// TQ_OK when the current device is an sm_100 GPU, else TQ_ERR_NO_DEVICE.
int device_status();
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream);

// The whole layer from bf16 X (decode sizes: one fused kernel).
struct LayerArgs {
  const uint32_t* signs = nullptr;  // randomized Hadamard sign masks [n_rht][K / 32], or null
  int n_rht = 1;
  const uint16_t* X;
  const uint16_t* L1t;
  const uint8_t* Wq;
  const float* s_w;
  const uint16_t* L2t;
  int M, N, K, r, had_block;
  uint16_t* Y;
  void* ws;  // status word at offset 0
};
// The decode layer sized for two CTAs per SM (clusters of K / 256 CTAs).
// Optional debug outputs: the activation codes [M][K] int8, the scales [M]
// and the integer sums [M][N] (sum_k qx qw) of the same launch.
bool layer_decode2_supported(int M, int N, int K, int r, int had_block);
cudaError_t launch_layer_decode2(const LayerArgs& a, cudaStream_t stream,
                                 int8_t* dbg_codes = nullptr, float* dbg_sx = nullptr,
                                 int32_t* dbg_acc = nullptr);

// Shared host helpers (defined in tq_gemm.cu).
int num_sms();
bool encode_tiled_2d(CUtensorMap* m, CUtensorMapDataType dtype, const void* ptr,
                     uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                     uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace tq
