// Shared definitions of the VSA kernels (device side) and their launchers.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace vsa {

// Bits of the device error word kept in the workspace.
enum : int { kErrTimeout = 1, kErrBadIndex = 2 };

constexpr int kCube = 64;  // tokens per 4x4x4 cube

// Raster token index of in-cube slot r of cube c (cube and slot numbering as
// documented in include/vsa.h).
__host__ __device__ __forceinline__ int cube_token(int c, int r, int H, int W) {
  const int Hc = H >> 2, Wc = W >> 2;
  const int ct = c / (Hc * Wc), ch = (c / Wc) % Hc, cw = c % Wc;
  const int t = 4 * ct + (r >> 4), h = 4 * ch + ((r >> 2) & 3), w = 4 * cw + (r & 3);
  return (t * H + h) * W + w;
}

struct GatherParams {
  const __nv_bfloat16* src[3];  // q, k, v raster [BH, N, D]
  __nv_bfloat16* dst[3];        // cube-major [BH, C, 64, D]; null: pool only for that tensor
  float* pool[3];               // [BH, C, D] cube means
  __nv_bfloat16* split[3];      // [3, BH, C, D] the means as three bf16 terms (hi, mid, lo)
  int BH, C, H, W, N;
};

struct CoarseParams {
  // 3-D maps (128-byte swizzle) over the bf16 three-term splits:
  //   tm_qs, tm_ks: [3 * BH][C][D], boxes of 128 rows x 64 channels;
  //   tm_vs: [3 * BH][C][D], boxes of 64 rows x 64 channels;
  //   tm_ps: [3 * BH][C][Cp], boxes of 128 rows x 64 columns.
  CUtensorMap tm_qs, tm_ks, tm_vs, tm_ps;
  float* s;            // [BH, C, C] scores
  __nv_bfloat16* psplit;  // [3, BH, C, Cp] coarse probabilities as bf16 terms (hi, mid, lo)
  int p_terms;         // terms of P written: 2 (the forward's output product), 3 (the backward's products)
  float* oc;           // [BH, C, D]
  float* oc_copy;      // optional second destination of oc (may be null)
  int Cp;              // C rounded up to a multiple of 8 (row pitch of psplit)
  int* err;
  unsigned long long wait_ns;
  int32_t* idx;        // [BH, C, kcap]
  int32_t* cnt;        // [BH, C]
  int BH, C, D, kcap;
  int topk;            // > 0: top-K; 0: top-p
  float top_p;
  int kmin, kmax;
  int do_select;       // 0: only probabilities (selection supplied by the caller)
  float scale;         // 1/sqrt(D)
};

struct FineParams {
  // tm_out: 5-D map over the raster out [BH][T][H][W][D] bf16; a box is one
  // cube's 4 x 4 x 4 tokens by 64 channels, in the 128-byte swizzle.
  // tm_k, tm_v: 2-D maps over the cube-major copies (rows of D bf16, 64 x 64 boxes).
  CUtensorMap tm_k, tm_v;
  CUtensorMap tm_out;
  const __nv_bfloat16* q;        // [BH, N, D] raster (query cubes are read from here)
  const int32_t* idx;            // [BH, C, kcap]
  const int32_t* cnt;            // [BH, C] or null (then every row has kcap ids)
  const int32_t* order;          // [BH * C] item order (schedule.cu), or null: items in index order
  const float* oc;               // [BH, C, D]
  const float* gate_c;           // [BH, N]
  const float* gate_f;           // [BH, N]
  __nv_bfloat16* out;            // [BH, N, D] or null
  float* out_fine;               // [BH, N, D] or null
  float* o_fine;                 // [BH, N, D] fp32 fine output saved for the backward pass, or null
  float* lse;                    // [BH, N] natural-log softmax denominators saved for the backward pass, or null
  int* err;
  unsigned long long wait_ns;
  int BH, C, H, W, N, kcap, n_items;
  float scale_log2;              // log2(e)/sqrt(D)
  int debug_stall;
};

// ---------------------------------------------------------------- backward pass
// Per-token preparation of the backward pass (one warp per query cube).
struct PrepParams {
  const __nv_bfloat16* dout;   // [BH, N, D] raster, gradient of the gated output
  const float* ofine;          // [BH, N, D] raster, fp32 fine output saved by the forward
  const float* lse;            // [BH, N] raster, natural-log softmax denominators saved by the forward
  const float* gate_c;         // [BH, N]
  const float* gate_f;         // [BH, N]
  const float* oc;             // [BH, C, D] coarse output (recomputed)
  __nv_bfloat16* do_cube;      // [BH, C, 64, D] gate_f * dout, cube-major (bf16)
  float* qstat;                // [BH, C, 2, 64]: lse * log2(e) and delta = bf16(gate_f dout) . ofine
  float* doc;                  // [BH, C, D] gradient of the coarse output
  __nv_bfloat16* docsplit;     // [3, BH, C, D] the same as three bf16 terms (hi, mid, lo)
  float* dlc;                  // [BH, C] doc . oc per cube
  float* dgate_c;              // [BH, N]
  float* dgate_f;              // [BH, N]
  int BH, C, H, W, N;
};

// Backward of the coarse attention on the pooled tokens: four C x C x D
// products per head on the tensor cores, each fp32 operand as three bf16
// terms (as in the forward's coarse products).
struct CoarseBwdParams {
  // 3-D maps [3 * BH][rows][cols] over three-term bf16 operands, 128-byte swizzle, boxes {64 cols, rows}:
  CUtensorMap tm_doc128, tm_vb128;         // dOc, vbar [C][D], 128-row boxes (dS product: A, B K-major)
  CUtensorMap tm_ds128;                    // dS [C][Cp], 128-row boxes (dqbar product: A K-major)
  CUtensorMap tm_kb64, tm_qb64, tm_doc64;  // kbar, qbar, dOc [C][D], 64-row boxes (B operands, N-major)
  CUtensorMap tm_ds64, tm_p64;             // dS, P [C][Cp], 64-row boxes (A MN-major: dkbar, dvbar products)
  const __nv_bfloat16* psplit;  // [3, BH, C, Cp] coarse probabilities (three terms), read by the dS epilogue
  __nv_bfloat16* dssplit;       // [3, BH, C, Cp] dS = P (dOc vbar^T - delta_c) as three terms (written)
  int Cp;
  const float* dlc;             // [BH, C]
  float* dqbar;                 // [BH, C, D] gradients of the pooled q, k, v
  float* dkbar;
  float* dvbar;
  int* err;
  unsigned long long wait_ns;
  int BH, C, D;
  float scale;                  // 1/sqrt(D)
};

// Transposed selection lists: for every KV cube, the query cubes that selected it.
struct TlistParams {
  const int32_t* idx;   // [BH, C, kcap]
  const int32_t* cnt;   // [BH, C] or null (every row holds kcap ids)
  uint32_t* bitmap;     // [BH, C, W32] bit i of row j: query cube i selected KV cube j
  int32_t* tcnt;        // [BH, C]
  int32_t* toff;        // [BH, C] absolute offsets into tlist
  int32_t* tlist;       // [BH * C * kcap] ascending query-cube ids per KV cube
  int* err;
  int BH, C, kcap, W32;
};

// Block-sparse fine attention backward (tcgen05). The dQ kernel walks query
// cubes over their selected KV cubes; the dK/dV kernel walks KV cubes over
// the query cubes that selected them.
struct BwdFineParams {
  // 2-D maps over cube-major copies [BH * C * 64][D] bf16, 64 x 64 boxes, 128-byte swizzle
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  // 5-D store maps over raster outputs [BH][T][H][W][D] bf16: dQ kernel tm_out0 = dq;
  // dK/dV kernel tm_out0 = dk, tm_out1 = dv
  CUtensorMap tm_out0, tm_out1;
  const int32_t* list;   // dQ: idx [BH * C, kcap]; dK/dV: the flat transposed lists
  const int32_t* cnt;    // dQ: counts or null (kcap each); dK/dV: tcnt
  const int32_t* off;    // dK/dV: toff; dQ: null
  const int32_t* order;  // [BH * C] item order (schedule.cu), or null: items in index order
  const float* qstat;    // [BH * C, 2, 64]
  const float* cpart0;   // [BH * C, D] coarse-path gradient rows: dQ kernel dq_bar; dK/dV kernel dk_bar
  const float* cpart1;   // dK/dV kernel dv_bar
  int* err;
  unsigned long long wait_ns;
  int BH, C, H, W, N, kcap, n_items;
  float scale_log2;      // log2(e) / sqrt(D)
  float scale;           // 1 / sqrt(D)
};

cudaError_t launch_gather(const GatherParams& p, int D, int num_sms, cudaStream_t st);
cudaError_t launch_coarse(const CoarseParams& p, cudaStream_t st);
cudaError_t launch_fine(const FineParams& p, int D, int grid, cudaStream_t st);
cudaError_t launch_bwd_prep(const PrepParams& p, int D, cudaStream_t st);
cudaError_t launch_coarse_bwd(const CoarseBwdParams& p, cudaStream_t st);
cudaError_t launch_tlists(const TlistParams& p, cudaStream_t st);
cudaError_t launch_fine_dq(const BwdFineParams& p, int D, int grid, cudaStream_t st);
cudaError_t launch_fine_dkv(const BwdFineParams& p, int D, int grid, cudaStream_t st);
cudaError_t launch_schedule(const int32_t* len, int32_t* order, int BH, int C, int maxlen, cudaStream_t st);
cudaError_t launch_l2_read(const void* buf, size_t bytes, int passes, int* status, int grid, cudaStream_t st);

}  // namespace vsa
