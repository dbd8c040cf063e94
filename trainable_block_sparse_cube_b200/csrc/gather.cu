// Cube gather and mean pool.
//
// "Faster Video Diffusion with Trainable Sparse Attention", "Approach":
// tokens are grouped into 4x4x4 cubes (one GPU tile per cube) and each cube
// is mean-pooled to one coarse token. This kernel reads each cube's 64 raster
// rows of q, k and v once, writes the fp32 mean of the 64 rows and, for k and
// v, copies the rows into one contiguous 64 x D block of the cube-major
// workspace (bit copy), from which the fine kernel streams them. The fine
// kernel reads q straight from its raster layout, so q's copy is written
// only when a plan asks for it for inspection.
//
// One warp per (tensor, head, cube) unit at a time: the grid is sized to
// about eight 256-thread blocks per SM and each warp strides over the units
// (tensor fastest, so the q, k and v of a cube go to neighbouring warps),
// which avoids the partial last wave of a one-unit-per-warp grid. A raster
// row of D bf16 is D*2 bytes; a lane moves 16 bytes, so D/8 lanes cover a row
// and a warp covers 32/(D/8) rows per step. Four consecutive w positions of a cube are contiguous in the
// raster layout (4*D*2 bytes), and every read and write is a full 16-byte
// vector. The pool sums are kept per lane in fp32 and combined with shuffles.
#include "vsa_common.cuh"

namespace vsa {

// One (tensor, head, cube) unit: the cube's 64 raster rows of tensor
// `tensor` -> its fp32 mean and three bf16 terms, and the cube-major copy
// when the tensor has one.
template <int D>
__device__ __forceinline__ void gather_pool_unit(const GatherParams& p, int tensor, int bh, int c, int sub, int chunk) {
  constexpr int LPR = D / 8;        // lanes per row
  constexpr int RPS = 32 / LPR;     // rows per warp step
  constexpr int STEPS = kCube / RPS;
  const __nv_bfloat16* src = p.src[tensor] + (size_t)bh * p.N * D + chunk * 8;
  const bool copy = p.dst[tensor] != nullptr;
  __nv_bfloat16* dst = copy ? p.dst[tensor] + ((size_t)bh * p.C + c) * kCube * D + chunk * 8 : nullptr;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  constexpr int U = STEPS < 8 ? STEPS : 8;
#pragma unroll
  for (int s0 = 0; s0 < STEPS; s0 += U) {
    int4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = (s0 + u) * RPS + sub;
      const int n = cube_token(c, r, p.H, p.W);
      v[u] = __ldg(reinterpret_cast<const int4*>(src + (size_t)n * D));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = (s0 + u) * RPS + sub;
      if (copy) *reinterpret_cast<int4*>(dst + (size_t)r * D) = v[u];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  if (sub == 0) {
    float* pool = p.pool[tensor] + ((size_t)bh * p.C + c) * D + chunk * 8;
    const float inv = 1.0f / kCube;
    *reinterpret_cast<float4*>(pool) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<float4*>(pool + 4) = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    // The same means as three bf16 terms (hi, mid, lo) for the tensor-core
    // coarse products, packed two per 32-bit word (lower element in the low half).
    uint32_t w[3][4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float x[2] = {acc[e] * inv, acc[e + 1] * inv};
      __nv_bfloat162 h[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        h[k] = __floats2bfloat162_rn(x[0], x[1]);
        const float2 back = __bfloat1622float2(h[k]);
        x[0] -= back.x;
        x[1] -= back.y;
      }
#pragma unroll
      for (int k = 0; k < 3; ++k) w[k][e / 2] = (uint32_t)__bfloat16_as_ushort(h[k].x) |
                                               ((uint32_t)__bfloat16_as_ushort(h[k].y) << 16);
    }
    const size_t plane = (size_t)p.BH * p.C * D;
    __nv_bfloat16* sp = p.split[tensor] + ((size_t)bh * p.C + c) * D + chunk * 8;
#pragma unroll
    for (int k = 0; k < 3; ++k)
      *reinterpret_cast<uint4*>(sp + k * plane) = make_uint4(w[k][0], w[k][1], w[k][2], w[k][3]);
  }
}

template <int D>
__global__ void __launch_bounds__(256) gather_pool_kernel(const GatherParams p) {
  constexpr int LPR = D / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, chunk = lane % LPR;
  const int units = 3 * p.BH * p.C;
  for (int unit = blockIdx.x * 8 + warp; unit < units; unit += gridDim.x * 8) {
    const int tensor = unit % 3, rest = unit / 3;
    const int bh = rest / p.C, c = rest - bh * p.C;
    gather_pool_unit<D>(p, tensor, bh, c, sub, chunk);
  }
}

cudaError_t launch_gather(const GatherParams& p, int D, int num_sms, cudaStream_t st) {
  const long long units = 3LL * p.BH * p.C;
  long long blocks = (units + 7) / 8;
  if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
  const dim3 grid((unsigned)blocks);
  if (D == 128)
    gather_pool_kernel<128><<<grid, 256, 0, st>>>(p);
  else
    gather_pool_kernel<64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace vsa
