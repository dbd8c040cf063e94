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
//   1. scores   s = qbar kbar^T / sqrt(D)       [BH, C, C]   (tiled SGEMM, 64 x 128 tiles)
//   2. select   row max / sum, exact K-th largest score by a 32-step radix
//               search on order-preserving integer keys (one warp per row,
//               keys in registers), ascending index lists with ties to the
//               lower id; top-p ranks the kmax best candidates and cuts at
//               the first prefix whose mass reaches p. Writes P over s.
//   3. output   Oc = P vbar                     [BH, C, D]   (tiled SGEMM, K split over
//               several CTAs per tile, partials added in a fixed order)
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

// ------------------------------------------------------------ fp32 GEMM tile
// One CTA computes a 64 x 128 tile of A . B over a range of K with 128
// threads, 8 x 8 outputs per thread (rows {4ty + i, 32 + 4ty + i}, columns
// {4tx + j, 64 + 4tx + j}), in steps of 16 along K staged through shared
// memory twice over so the global loads of step k+1 overlap the FMAs of
// step k.
//   A: row-major [M x K] (element (m, k) at A[m * lda + k]).
//   B: B_KMAJOR ? row-major [N x K] (element (n, k) at B[n * ldb + k])
//               : row-major [K x N] (element (k, n) at B[k * ldb + n]).
constexpr int kGM = 64, kGN = 128, kGK = 16, kGThreads = 128;

struct GemmSmem {
  float a[2][kGK][kGM + 4];  // [k][m]
  float b[2][kGK][kGN + 4];  // [k][n]
};

template <bool B_KMAJOR>
struct GemmTile {
  const float* A;
  const float* B;
  int lda, ldb, M, N;
  bool a_vec;  // A rows 16-byte aligned: float4 loads
  float ra[8], rb[16];

  __device__ __forceinline__ void load(int m0, int n0, int k0, int k_end) {
    const int tid = threadIdx.x;
    {  // A: row m0 + tid / 2, k0 + 8 (tid % 2) .. + 7
      const int m = m0 + (tid >> 1), kb = k0 + (tid & 1) * 8;
      const float* src = A + (size_t)m * lda + kb;
      if (a_vec && m < M && kb + 8 <= k_end) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        const float4 y = *reinterpret_cast<const float4*>(src + 4);
        ra[0] = x.x; ra[1] = x.y; ra[2] = x.z; ra[3] = x.w;
        ra[4] = y.x; ra[5] = y.y; ra[6] = y.z; ra[7] = y.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) ra[e] = (m < M && kb + e < k_end) ? src[e] : 0.f;
      }
    }
    if (B_KMAJOR) {  // B: row n0 + tid, k0 .. k0 + 15
      const int n = n0 + tid;
      const float* src = B + (size_t)n * ldb + k0;
      if (n < N && k0 + 16 <= k_end) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 x = *reinterpret_cast<const float4*>(src + 4 * q);
          rb[4 * q] = x.x; rb[4 * q + 1] = x.y; rb[4 * q + 2] = x.z; rb[4 * q + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) rb[e] = (n < N && k0 + e < k_end) ? src[e] : 0.f;
      }
    } else {  // B: row k0 + tid / 8, columns n0 + 16 (tid % 8) .. + 15
      const int k = k0 + (tid >> 3), nb = n0 + (tid & 7) * 16;
      const float* src = B + (size_t)k * ldb + nb;
      if (k < k_end && nb + 16 <= N) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 x = *reinterpret_cast<const float4*>(src + 4 * q);
          rb[4 * q] = x.x; rb[4 * q + 1] = x.y; rb[4 * q + 2] = x.z; rb[4 * q + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) rb[e] = (k < k_end && nb + e < N) ? src[e] : 0.f;
      }
    }
  }

  __device__ __forceinline__ void store(GemmSmem& sm, int buf) const {
    const int tid = threadIdx.x;
    const int m = tid >> 1, kb = (tid & 1) * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) sm.a[buf][kb + e][m] = ra[e];
    if (B_KMAJOR) {
#pragma unroll
      for (int e = 0; e < 16; ++e) sm.b[buf][e][tid] = rb[e];
    } else {
      const int k = tid >> 3, nb = (tid & 7) * 16;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(&sm.b[buf][k][nb + 4 * q]) =
            make_float4(rb[4 * q], rb[4 * q + 1], rb[4 * q + 2], rb[4 * q + 3]);
    }
  }

  // acc += A[m0.., k_begin..k_end) . B[.., n0..]
  __device__ __forceinline__ void run(GemmSmem& sm, int m0, int n0, int k_begin, int k_end, float (&acc)[8][8]) {
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    int buf = 0;
    load(m0, n0, k_begin, k_end);
    store(sm, 0);
    __syncthreads();
    for (int k0 = k_begin; k0 < k_end; k0 += kGK) {
      const bool more = k0 + kGK < k_end;
      if (more) load(m0, n0, k0 + kGK, k_end);
#pragma unroll
      for (int kk = 0; kk < kGK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&sm.a[buf][kk][4 * ty]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sm.a[buf][kk][32 + 4 * ty]);
        const float4 b0 = *reinterpret_cast<const float4*>(&sm.b[buf][kk][4 * tx]);
        const float4 b1 = *reinterpret_cast<const float4*>(&sm.b[buf][kk][64 + 4 * tx]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      if (more) store(sm, buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
};

// Row and column of accumulator (i, j) of this thread within the 64 x 128 tile.
__device__ __forceinline__ int tile_row(int i) { return (i < 4 ? 0 : 32) + 4 * (threadIdx.x >> 4) + (i & 3); }
__device__ __forceinline__ int tile_col(int j) { return (j < 4 ? 0 : 64) + 4 * (threadIdx.x & 15) + (j & 3); }

// ------------------------------------------------------------ 1. scores
__global__ void __launch_bounds__(kGThreads) coarse_scores_kernel(const CoarseParams p) {
  __shared__ __align__(16) GemmSmem sm;
  const int C = p.C, D = p.D;
  const int bh = blockIdx.z, m0 = blockIdx.y * kGM, n0 = blockIdx.x * kGN;
  GemmTile<true> g{p.qpool + (size_t)bh * C * D, p.kpool + (size_t)bh * C * D, D, D, C, C, true};
  float acc[8][8] = {};
  g.run(sm, m0, n0, 0, D, acc);
  float* S = p.s + (size_t)bh * C * C;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + tile_row(i);
    if (r >= C) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = n0 + tile_col(j);
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

// Exact Kt-th largest key of the warp's row: the largest T with
// #{key >= T} >= Kt, by an MSB-first search over the 32 key bits. For
// Kt <= 32 the minimum of the lanes' maxima is a lower bound of the answer
// (the 32 lane maxima are Kt or more keys at or above it), so the search runs
// over the few keys at or above that bound, compacted into `cand` (kCandCap
// per warp); it falls back to all keys when there are too many of them.
constexpr int kCandCap = 256;
template <int PER>
__device__ __forceinline__ uint32_t kth_largest(const uint32_t (&key)[PER], int C, int Kt, uint32_t* cand) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  if (Kt <= 32) {
    uint32_t lmax = 0;
    bool any = false;
#pragma unroll
    for (int u = 0; u < PER; ++u)
      if (lane + 32 * u < C) {
        lmax = max(lmax, key[u]);
        any = true;
      }
    const uint32_t lo = __reduce_min_sync(0xffffffffu, any ? lmax : 0xffffffffu);
    unsigned nl = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) nl += (key[u] >= lo);
    const int n = (int)__reduce_add_sync(0xffffffffu, nl);
    if (n <= kCandCap) {
      int pos = 0;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const bool t = key[u] >= lo;
        const unsigned tb = __ballot_sync(0xffffffffu, t);
        if (t) cand[pos + __popc(tb & lt_mask)] = key[u];
        pos += __popc(tb);
      }
      __syncwarp();
      uint32_t ck[kCandCap / 32];
#pragma unroll
      for (int i = 0; i < kCandCap / 32; ++i) ck[i] = (lane + 32 * i < n) ? cand[lane + 32 * i] : 0u;
      __syncwarp();
      uint32_t T = 0;
      for (int b = 31; b >= 0; --b) {
        const uint32_t c = T | (1u << b);
        unsigned cnt = 0;
#pragma unroll
        for (int i = 0; i < kCandCap / 32; ++i) cnt += (ck[i] >= c);
        if ((int)__reduce_add_sync(0xffffffffu, cnt) >= Kt) T = c;
      }
      return T;
    }
  }
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t c = T | (1u << b);
    unsigned cnt = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) cnt += (key[u] >= c);
    if ((int)__reduce_add_sync(0xffffffffu, cnt) >= Kt) T = c;
  }
  return T;
}

// TOPK: fixed top-K (no top-p scratch, fewer registers, more warps per SM).
template <int PER, bool TOPK>
__global__ void __launch_bounds__(256, TOPK ? 3 : 1) coarse_select_kernel(const CoarseParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ uint32_t cand_all[8][kCandCap];
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
    // T is the Kt-th largest key exactly.
    const uint32_t T = kth_largest<PER>(key, C, Kt, cand_all[warp]);
    unsigned gtl = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) gtl += (key[u] > T);
    const int need = Kt - (int)__reduce_add_sync(0xffffffffu, gtl);  // ids equal to T to take, lowest first

    int32_t* irow = p.idx + (size_t)row * p.kcap;
    int n_out;
    if (TOPK) {
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
// Oc = P . vbar with K (the C key cubes) split into p.splits ranges: each CTA
// writes the partial product of its range, and the last CTA of a tile (an
// atomic arrival count) adds the partials in split order, so the sum is the
// same on every run.
__global__ void __launch_bounds__(kGThreads) coarse_output_kernel(const CoarseParams p) {
  __shared__ __align__(16) GemmSmem sm;
  __shared__ int last;
  const int C = p.C, D = p.D, S = p.splits;
  const int bh = blockIdx.z, split = blockIdx.y, mt = blockIdx.x, m0 = mt * kGM;
  const int kper = (((C + S - 1) / S) + kGK - 1) / kGK * kGK;
  const int kb = split * kper, ke = min(C, kb + kper);
  GemmTile<false> g{p.s + (size_t)bh * C * C, p.vpool + (size_t)bh * C * D, C, D, C, D, (C & 3) == 0};
  float acc[8][8] = {};
  if (kb < ke) g.run(sm, m0, 0, kb, ke, acc);
  float* dst = S == 1 ? p.oc + (size_t)bh * C * D : p.opart + ((size_t)split * p.BH + bh) * C * D;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + tile_row(i);
    if (r >= C) continue;
#pragma unroll
    for (int jb = 0; jb < 8; jb += 4) {
      const int c = tile_col(jb);
      if (c < D) *reinterpret_cast<float4*>(dst + (size_t)r * D + c) =
                     make_float4(acc[i][jb], acc[i][jb + 1], acc[i][jb + 2], acc[i][jb + 3]);
    }
  }
  if (S == 1) {
    if (p.oc_copy) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = m0 + tile_row(i);
        if (r >= C) continue;
#pragma unroll
        for (int jb = 0; jb < 8; jb += 4) {
          const int c = tile_col(jb);
          if (c < D) *reinterpret_cast<float4*>(p.oc_copy + ((size_t)bh * C + r) * D + c) =
                         make_float4(acc[i][jb], acc[i][jb + 1], acc[i][jb + 2], acc[i][jb + 3]);
        }
      }
    }
    return;
  }
  __threadfence();
  __syncthreads();
  int* cnt = p.tile_cnt + bh * gridDim.x + mt;
  if (threadIdx.x == 0) last = (atomicAdd(cnt, 1) == S - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  // Sum the partials of the tile's rows in split order (16 bytes per thread per step).
  const int rows = min(kGM, C - m0), vecs = rows * (D / 4);
  for (int v = threadIdx.x; v < vecs; v += kGThreads) {
    const size_t o = ((size_t)bh * C + m0 + v / (D / 4)) * D + (v % (D / 4)) * 4;
    float4 t = __ldcg(reinterpret_cast<const float4*>(p.opart + o));
    for (int s2 = 1; s2 < S; ++s2) {
      const float4 u = __ldcg(reinterpret_cast<const float4*>(p.opart + (size_t)s2 * p.BH * C * D + o));
      t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
    }
    *reinterpret_cast<float4*>(p.oc + o) = t;
    if (p.oc_copy) *reinterpret_cast<float4*>(p.oc_copy + o) = t;
  }
  if (threadIdx.x == 0) *cnt = 0;  // ready for the next run
}

template <int PER>
cudaError_t launch_select(const CoarseParams& p, cudaStream_t st) {
  const int rows = p.BH * p.C;
  if (!p.do_select || p.topk > 0) {
    coarse_select_kernel<PER, true><<<(rows + 7) / 8, 256, 0, st>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)8 * p.kmax * 16;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(coarse_select_kernel<PER, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  coarse_select_kernel<PER, false><<<(rows + 7) / 8, 256, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_coarse(const CoarseParams& p, cudaStream_t st) {
  const int mtiles = (p.C + kGM - 1) / kGM, ntiles = (p.C + kGN - 1) / kGN;
  coarse_scores_kernel<<<dim3(ntiles, mtiles, p.BH), kGThreads, 0, st>>>(p);
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
  coarse_output_kernel<<<dim3(mtiles, p.splits, p.BH), kGThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace vsa
