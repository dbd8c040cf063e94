// Coarse stage: dense cube-to-cube attention on the pooled tokens and the
// per-query-cube selection of critical KV cubes.
//
// "Faster Video Diffusion with Trainable Sparse Attention", "Approach": a
// coarse cube-to-cube dense attention selects the top-K critical cubes and
// outputs a coarse context. "Improving Video Sparse Attention with
// Fine-grained Router and Sparse Rebasing", "Abstract (arXiv)": each query
// may keep a variable number of key-value blocks; here that is the top-p
// rule documented in include/vsa.h.
//
// Three launches per call, all in fp32 on the CUDA cores (the scores decide
// integer selections, so they are kept in fp32 rather than bf16):
//   1. scores   s = qbar kbar^T / sqrt(D)       [BH, C, C]   (tiled SGEMM)
//   2. select   row max / sum, exact K-th largest score by a 32-step radix
//               search on order-preserving integer keys (one warp per row,
//               keys in registers), ascending index lists with ties to the
//               lower id; top-p ranks the kmax best candidates and cuts at
//               the first prefix whose mass reaches p. Writes P over s.
//   3. output   Oc = P vbar                     [BH, C, D]   (tiled SGEMM)
#include "vsa_common.cuh"

namespace vsa {

namespace {

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Larger float -> larger unsigned key (sign-magnitude to biased order).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ 1. scores
__global__ void __launch_bounds__(256) coarse_scores_kernel(const CoarseParams p) {
  __shared__ __align__(16) float As[16][68];
  __shared__ __align__(16) float Bs[16][68];
  const int C = p.C, D = p.D;
  const int bh = blockIdx.z, row0 = blockIdx.y * 64, col0 = blockIdx.x * 64;
  const float* A = p.qpool + (size_t)bh * C * D;
  const float* Bm = p.kpool + (size_t)bh * C * D;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lk = (tid & 3) * 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < D; k0 += 16) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (row0 + lr < C) a = *reinterpret_cast<const float4*>(A + (size_t)(row0 + lr) * D + k0 + lk);
    if (col0 + lr < C) b = *reinterpret_cast<const float4*>(Bm + (size_t)(col0 + lr) * D + k0 + lk);
    __syncthreads();
    As[lk + 0][lr] = a.x; As[lk + 1][lr] = a.y; As[lk + 2][lr] = a.z; As[lk + 3][lr] = a.w;
    Bs[lk + 0][lr] = b.x; Bs[lk + 1][lr] = b.y; Bs[lk + 2][lr] = b.z; Bs[lk + 3][lr] = b.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
  }
  float* S = p.s + (size_t)bh * C * C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty * 4 + i;
    if (r >= C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = col0 + tx * 4 + j;
      if (c < C) S[(size_t)r * C + c] = acc[i][j] * p.scale;
    }
  }
}

// ------------------------------------------------------------ 2. select
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Per-warp scratch for top-p ranking: kmax entries of (id, key, weight) and
// the weights in rank order.
struct TopPScratch {
  int* id;
  uint32_t* key;
  float* w;
  float* sorted;
};

template <int PER>
__global__ void __launch_bounds__(256) coarse_select_kernel(const CoarseParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= p.BH * p.C) return;
  const int C = p.C;
  float* srow = p.s + (size_t)row * C;
  const uint32_t lt_mask = (1u << lane) - 1u;

  uint32_t key[PER];
  float m = -INFINITY;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int j = lane + 32 * u;
    const float s = (j < C) ? srow[j] : -INFINITY;
    key[u] = (j < C) ? order_key(s) : 0u;
    m = fmaxf(m, s);
  }
  m = warp_max(m);
  const float mb = m * kLog2e;
  float l = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u)
    if (lane + 32 * u < C) l += fast_exp2(fmaf(key_value(key[u]), kLog2e, -mb));
  l = warp_sum(l);

  if (p.do_select) {
    const int Kt = p.topk > 0 ? p.topk : p.kmax;
    // Largest T with #{key >= T} >= Kt: T is the Kt-th largest key exactly.
    uint32_t T = 0;
    for (int b = 31; b >= 0; --b) {
      const uint32_t cand = T | (1u << b);
      unsigned cntl = 0;
#pragma unroll
      for (int u = 0; u < PER; ++u) cntl += (key[u] >= cand);
      if ((int)__reduce_add_sync(0xffffffffu, cntl) >= Kt) T = cand;
    }
    unsigned gtl = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) gtl += (key[u] > T);
    const int need = Kt - (int)__reduce_add_sync(0xffffffffu, gtl);  // ids equal to T to take, lowest first

    int32_t* irow = p.idx + (size_t)row * p.kcap;
    int n_out;
    if (p.topk > 0) {
      int pos = 0, eq_seen = 0;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int j = lane + 32 * u;
        const bool is_eq = (key[u] == T) && (j < C);
        const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
        const bool take = (key[u] > T) || (is_eq && eq_seen + __popc(eqb & lt_mask) < need);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (take) irow[pos + __popc(tb & lt_mask)] = j;
        pos += __popc(tb);
        eq_seen += __popc(eqb);
      }
      n_out = Kt;
    } else {
      const int kmax = p.kmax;
      TopPScratch sc;
      uint8_t* base = dyn + (size_t)warp * kmax * 16;
      sc.id = reinterpret_cast<int*>(base);
      sc.key = reinterpret_cast<uint32_t*>(base + kmax * 4);
      sc.w = reinterpret_cast<float*>(base + kmax * 8);
      sc.sorted = reinterpret_cast<float*>(base + kmax * 12);
      int pos = 0, eq_seen = 0;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int j = lane + 32 * u;
        const bool is_eq = (key[u] == T) && (j < C);
        const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
        const bool take = (key[u] > T) || (is_eq && eq_seen + __popc(eqb & lt_mask) < need);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (take) {
          const int q = pos + __popc(tb & lt_mask);
          sc.id[q] = j;
          sc.key[q] = key[u];
          sc.w[q] = fast_exp2(fmaf(key_value(key[u]), kLog2e, -mb));
        }
        pos += __popc(tb);
        eq_seen += __popc(eqb);
      }
      __syncwarp();
      // Rank = number of candidates ahead in (score desc, id asc) order.
      for (int c = lane; c < Kt; c += 32) {
        const uint32_t kc = sc.key[c];
        int r = 0;
        for (int o = 0; o < Kt; ++o) {
          const uint32_t ko = sc.key[o];
          r += (ko > kc) || (ko == kc && o < c);  // candidates are stored in ascending id
        }
        sc.sorted[r] = sc.w[c];
        sc.id[c] = sc.id[c] | (r << 16);  // pack rank above the id (ids < 65536)
      }
      __syncwarp();
      // First rank whose cumulative weight reaches top_p * l.
      const int CH = (Kt + 31) / 32;
      const int b0 = lane * CH, b1 = min(b0 + CH, Kt);
      float part = 0.f;
      for (int r = b0; r < b1; ++r) part += sc.sorted[r];
      float incl = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      float run = incl - part;
      const float target = p.top_p * l;
      int first = 0x7fffffff;
      for (int r = b0; r < b1; ++r) {
        run += sc.sorted[r];
        if (run >= target) { first = r; break; }
      }
      first = __reduce_min_sync(0xffffffffu, first);
      int nsel = (first == 0x7fffffff) ? Kt : first + 1;
      nsel = max(nsel, p.kmin);
      nsel = min(nsel, Kt);
      // Emit candidates with rank < nsel in ascending id order.
      int opos = 0;
      for (int c0 = 0; c0 < Kt; c0 += 32) {
        const int c = c0 + lane;
        int packed = (c < Kt) ? sc.id[c] : 0;
        const bool take = (c < Kt) && ((packed >> 16) < nsel);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (take) irow[opos + __popc(tb & lt_mask)] = packed & 0xffff;
        opos += __popc(tb);
      }
      n_out = nsel;
    }
    for (int c = n_out + lane; c < p.kcap; c += 32) irow[c] = -1;
    if (lane == 0) p.cnt[row] = n_out;
  }
  // Probabilities over the scores (read back by the output SGEMM).
  const float inv_l = 1.0f / l;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int j = lane + 32 * u;
    if (j < C) srow[j] = fast_exp2(fmaf(key_value(key[u]), kLog2e, -mb)) * inv_l;
  }
}

// ------------------------------------------------------------ 3. output
__global__ void __launch_bounds__(256) coarse_output_kernel(const CoarseParams p) {
  __shared__ __align__(16) float As[16][68];  // [j][row]
  __shared__ __align__(16) float Bs[16][68];  // [j][d]
  const int C = p.C, D = p.D;
  const int bh = blockIdx.z, row0 = blockIdx.y * 64, d0 = blockIdx.x * 64;
  const float* P = p.s + (size_t)bh * C * C;
  const float* V = p.vpool + (size_t)bh * C * D;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lk = (tid & 3) * 4;   // A tile: row, j offset
  const int bj = tid >> 4, bd = (tid & 15) * 4;  // B tile: j, d offset
  float acc[4][4] = {};
  for (int k0 = 0; k0 < C; k0 += 16) {
    float a[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = row0 + lr, j = k0 + lk + e;
      a[e] = (r < C && j < C) ? P[(size_t)r * C + j] : 0.f;
    }
    float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
    if (k0 + bj < C) b = *reinterpret_cast<const float4*>(V + (size_t)(k0 + bj) * D + d0 + bd);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 4; ++e) As[lk + e][lr] = a[e];
    *reinterpret_cast<float4*>(&Bs[bj][bd]) = b;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty * 4 + i;
    if (r >= C) continue;
    const size_t o = ((size_t)bh * C + r) * D + d0 + tx * 4;
    const float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    *reinterpret_cast<float4*>(p.oc + o) = v;
    if (p.oc_copy) *reinterpret_cast<float4*>(p.oc_copy + o) = v;
  }
}

template <int PER>
cudaError_t launch_select(const CoarseParams& p, cudaStream_t st) {
  const int rows = p.BH * p.C;
  const size_t smem = (p.do_select && p.topk == 0) ? (size_t)8 * p.kmax * 16 : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(coarse_select_kernel<PER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  coarse_select_kernel<PER><<<(rows + 7) / 8, 256, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_coarse(const CoarseParams& p, cudaStream_t st) {
  const int tiles = (p.C + 63) / 64;
  coarse_scores_kernel<<<dim3(tiles, tiles, p.BH), 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int per = (p.C + 31) / 32;
  if (per <= 1) e = launch_select<1>(p, st);
  else if (per <= 2) e = launch_select<2>(p, st);
  else if (per <= 4) e = launch_select<4>(p, st);
  else if (per <= 8) e = launch_select<8>(p, st);
  else if (per <= 16) e = launch_select<16>(p, st);
  else if (per <= 24) e = launch_select<24>(p, st);
  else if (per <= 32) e = launch_select<32>(p, st);
  else if (per <= 40) e = launch_select<40>(p, st);
  else if (per <= 48) e = launch_select<48>(p, st);
  else if (per <= 64) e = launch_select<64>(p, st);
  else if (per <= 96) e = launch_select<96>(p, st);
  else e = launch_select<128>(p, st);
  if (e != cudaSuccess) return e;
  coarse_output_kernel<<<dim3(p.D / 64, tiles, p.BH), 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace vsa
