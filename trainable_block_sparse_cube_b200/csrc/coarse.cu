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
// Three launches per call. The scores decide integer selections, so both
// products keep fp32 accuracy; they run on the tensor cores by writing every
// fp32 operand x as three bf16 terms x = hi + mid + lo (8 significant bits
// each, |x - hi - mid - lo| <= 2^-25 |x|) and summing the six products
// hi.hi, hi.mid, mid.hi, mid.mid, hi.lo, lo.hi in fp32 tensor memory; the
// dropped ones are below 2^-24 relative.
//   1. scores   s = qbar kbar^T / sqrt(D)       [BH, C, C]   (tcgen05, 128 x 128 tiles)
//   2. select   one warp per row, the row's scores as order-preserving
//               uint32 keys: row max and sum, the probabilities P written as
//               bf16 terms (hi and mid for the forward's output product, also
//               lo when the backward's products need them), then the
//               selection. Top-K <= 32 with C <= 1024 (own kernel): the row
//               stays in registers; the minimum of the lanes' maxima bounds
//               the K-th largest key from below, each lane places its keys at
//               or above it through a prefix sum over the lanes, an MSB-first
//               count search over those candidates finds the K-th largest,
//               and the ids go out through two bitmaps (above it, equal to it)
//               in ascending order. Larger K or C, or more than 256
//               candidates, search over all keys in shared memory. Top-p (own
//               kernel): the exact kmax-th largest key by the same search,
//               the kmax candidates ranked by (score desc, id asc) and cut at
//               the first prefix whose mass reaches p, clamped to
//               [kmin, kmax]. Lists are ascending, ties go to the lower id.
//   3. output   Oc = P vbar                     [BH, C, D]   (tcgen05, 128 x D tiles)
#include "sm100_ptx.cuh"
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

constexpr int kCandCap = 256;

// MSB-first search for the Kt-th largest of the row's C keys (in shared
// memory): the largest T with #{key >= T} >= Kt.
__device__ __forceinline__ uint32_t kth_largest(const uint32_t* keys, int C, int Kt, int lane) {
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t c = T | (1u << b);
    unsigned cnt = 0;
    for (int j = lane; j < C; j += 32) cnt += (keys[j] >= c);
    if ((int)__reduce_add_sync(0xffffffffu, cnt) >= Kt) T = c;
  }
  return T;
}

// Loads row `row` of the scores into shared memory as order-preserving keys,
// then writes its softmax probabilities as three bf16 terms (zero in the
// padding columns C .. Cp-1), the A operand of the output product. Returns
// the row max in log2 units (mb), the row sum l and this lane's largest key.
__device__ __forceinline__ void row_softmax(const CoarseParams& p, int row, uint32_t* keys, int lane, float& mb,
                                            float& l, uint32_t& lkmax) {
  const int C = p.C;
  const float* srow = p.s + (size_t)row * C;
  float lm = -INFINITY;
  lkmax = 0;
  for (int j0 = 0; j0 < C; j0 += 256) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + lane + 32 * u;
      v[u] = j < C ? srow[j] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + lane + 32 * u;
      if (j < C) {
        const uint32_t k = order_key(v[u]);
        keys[j] = k;
        lkmax = max(lkmax, k);
        lm = fmaxf(lm, v[u]);
      }
    }
  }
  mb = warp_max(lm) * kLog2e;
  __syncwarp();
  float ls = 0.f;
  for (int j = lane; j < C; j += 32) ls += fast_exp2(fmaf(key_value(keys[j]), kLog2e, -mb));
  l = warp_sum(ls);
  const float inv_l = 1.0f / l;
  const size_t plane = (size_t)p.BH * C * p.Cp;
  __nv_bfloat16* prow = p.psplit + (size_t)row * p.Cp;
  for (int j = lane; j < p.Cp; j += 32) {
    const float x = j < C ? fast_exp2(fmaf(key_value(keys[j]), kLog2e, -mb)) * inv_l : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 md = __float2bfloat16_rn(r1);
    prow[j] = h;
    prow[plane + j] = md;
    if (p.p_terms > 2) prow[2 * plane + j] = __float2bfloat16_rn(r1 - __bfloat162float(md));
  }
}

// Row `row` of the scores in registers for C <= 1024: lane t holds columns
// 64u + 2t and 64u + 2t + 1 (u < 16) in v[2u], v[2u + 1]; -inf past C.
__device__ __forceinline__ void load_row_regs(const CoarseParams& p, int row, int lane, float (&v)[32]) {
  const int C = p.C;
  const float* srow = p.s + (size_t)row * C;
  if ((C & 1) == 0) {  // even C: every row starts 8-byte aligned and a pair never straddles C
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = 64 * u + 2 * lane;
      const float2 x = j < C ? *reinterpret_cast<const float2*>(srow + j) : make_float2(-INFINITY, -INFINITY);
      v[2 * u] = x.x;
      v[2 * u + 1] = x.y;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = 64 * u + 2 * lane;
      v[2 * u] = j < C ? srow[j] : -INFINITY;
      v[2 * u + 1] = j + 1 < C ? srow[j + 1] : -INFINITY;
    }
  }
}

// The probabilities v * inv_l of a register-resident row (load_row_regs
// layout) as TERMS bf16 terms (hi, mid[, lo]), written as bf16 pairs.
template <int TERMS>
__device__ __forceinline__ void store_p_terms(const CoarseParams& p, int row, int lane, const float (&v)[32],
                                              float inv_l) {
  const size_t plane = (size_t)p.BH * p.C * p.Cp;
  __nv_bfloat16* prow = p.psplit + (size_t)row * p.Cp;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int j = 64 * u + 2 * lane;
    if (j < p.Cp) {  // Cp is a multiple of 8: the pair j, j + 1 lies inside the row
      float x0 = v[2 * u] * inv_l, x1 = v[2 * u + 1] * inv_l;
#pragma unroll
      for (int t = 0; t < TERMS; ++t) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
        *reinterpret_cast<__nv_bfloat162*>(prow + t * plane + j) = h;
        if (t + 1 < TERMS) {
          const float2 back = __bfloat1622float2(h);
          x0 -= back.x;
          x1 -= back.y;
        }
      }
    }
  }
}

// Softmax of a register-resident row (load_row_regs layout) with row max lm:
// writes the probabilities' terms as bf16 pairs, returns the row max in log2
// units (mb) and the row sum l. v is overwritten with the numerators.
template <bool SPLIT_TERMS>
__device__ __forceinline__ void softmax_store_regs(const CoarseParams& p, int row, int lane, float (&v)[32], float lm,
                                                   float& mb, float& l) {
  mb = warp_max(lm) * kLog2e;
  float ls = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    v[e] = fast_exp2(fmaf(v[e], kLog2e, -mb));  // -inf (padding) -> 0
    ls += v[e];
  }
  l = warp_sum(ls);
  const float inv_l = 1.0f / l;
  if (SPLIT_TERMS) {  // one copy of the store loop per term count: no wasted third term in the forward
    if (p.p_terms > 2) store_p_terms<3>(p, row, lane, v, inv_l);
    else store_p_terms<2>(p, row, lane, v, inv_l);
  } else {  // one loop for either count (fewer registers)
    const size_t plane = (size_t)p.BH * p.C * p.Cp;
    __nv_bfloat16* prow = p.psplit + (size_t)row * p.Cp;
    const int terms = p.p_terms;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = 64 * u + 2 * lane;
      if (j < p.Cp) {
        float x0 = v[2 * u] * inv_l, x1 = v[2 * u + 1] * inv_l;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
          const float2 back = __bfloat1622float2(h);
          x0 -= back.x;
          x1 -= back.y;
          if (t < terms) *reinterpret_cast<__nv_bfloat162*>(prow + t * plane + j) = h;
        }
      }
    }
  }
}

// row_softmax for C <= 1024 with the row in registers, so every score is read
// once and every exponential computed once; the keys still go to shared
// memory for the selection.
__device__ __forceinline__ void row_softmax_regs(const CoarseParams& p, int row, uint32_t* keys, int lane, float& mb,
                                                 float& l, uint32_t& lkmax) {
  const int C = p.C;
  float v[32];
  load_row_regs(p, row, lane, v);
  float lm = -INFINITY;
  lkmax = 0;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int j = 64 * u + 2 * lane;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (j + h < C) {
        const uint32_t k = order_key(v[2 * u + h]);
        keys[j + h] = k;
        lkmax = max(lkmax, k);
        lm = fmaxf(lm, v[2 * u + h]);
      }
  }
  softmax_store_regs<false>(p, row, lane, v, lm, mb, l);
  __syncwarp();
}

// Top-K emission for Kt <= 32 from the candidates (keys at or above the lower
// bound lo, with their ids, in ascending id order, NS slots per lane): the
// Kt-th largest key T by the MSB-first search below the bits that lo and the
// row maximum hi share (T lies between them), then the ids of the keys above
// T and of the lowest-id keys equal to T, ascending.
template <int NS>
__device__ __forceinline__ void topk_from_candidates(const uint32_t* ckey, const int* cidx, int n, int Kt, uint32_t lo,
                                                     uint32_t hi, int32_t* irow) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t ck[NS];
  int cj[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int e = lane + 32 * i;
    ck[i] = e < n ? ckey[e] : 0u;
    cj[i] = e < n ? cidx[e] : 0;
  }
  uint32_t T = lo;
  if (lo != hi) {
    const int hb = 31 - __clz(lo ^ hi);
    T = hi & ~((2u << hb) - 1u);
    for (int b = hb; b >= 0; --b) {
      const uint32_t c = T | (1u << b);
      unsigned cnt = 0;
#pragma unroll
      for (int i = 0; i < NS; ++i) cnt += (ck[i] >= c);
      if ((int)__reduce_add_sync(0xffffffffu, cnt) >= Kt) T = c;
    }
  }
  unsigned gt = 0;
#pragma unroll
  for (int i = 0; i < NS; ++i) gt += (ck[i] > T);
  const int need = Kt - (int)__reduce_add_sync(0xffffffffu, gt);
  int pos = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const bool valid = lane + 32 * i < n;
    const bool is_eq = valid && ck[i] == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take = valid && (ck[i] > T || (is_eq && eq_seen + __popc(eqb & lt_mask) < need));
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) irow[pos + __popc(tb & lt_mask)] = cj[i];
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

// Warp-wide inclusive prefix sum.
__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Top-K emission for Kt <= 32 and C <= 1024 from candidates in any order
// (keys at or above the lower bound lo with their ids, NS slots per lane):
// the Kt-th largest key T by the MSB-first search below the bits that lo and
// the row maximum hi share, then the ids through two 32-word bitmaps in
// shared memory (bm[0..31]: keys above T, bm[32..63]: keys equal to T). Word
// w holds ids 32w..32w+31, so lane w emits its word's ids in ascending order
// at the prefix of the words before it, and the ties taken are the lowest ids.
template <int NS>
__device__ __forceinline__ void topk_bitmap_emit(const uint32_t* ckey, const int* cidx, int n, int Kt, uint32_t lo,
                                                 uint32_t hi, uint32_t* bm, int32_t* irow) {
  const int lane = threadIdx.x & 31;
  uint32_t ck[NS];
  int cj[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int e = lane + 32 * i;
    ck[i] = e < n ? ckey[e] : 0u;
    cj[i] = e < n ? cidx[e] : 0;
  }
  uint32_t T = lo;
  if (lo != hi) {
    const int hb = 31 - __clz(lo ^ hi);
    T = hi & ~((2u << hb) - 1u);
    for (int b = hb; b >= 0; --b) {
      const uint32_t c = T | (1u << b);
      unsigned cnt = 0;
#pragma unroll
      for (int i = 0; i < NS; ++i) cnt += (ck[i] >= c);
      if ((int)__reduce_add_sync(0xffffffffu, cnt) >= Kt) T = c;
    }
  }
  bm[lane] = 0u;
  bm[32 + lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NS; ++i)
    if (lane + 32 * i < n && ck[i] >= T) atomicOr(&bm[(ck[i] > T ? 0 : 32) + (cj[i] >> 5)], 1u << (cj[i] & 31));
  __syncwarp();
  const uint32_t g = bm[lane], q = bm[32 + lane];
  const int need = Kt - (int)__reduce_add_sync(0xffffffffu, (unsigned)__popc(g));
  const int neq = __popc(q);
  int take = min(max(need - (warp_incl_scan(neq, lane) - neq), 0), neq);
  uint32_t sel = g, rest = q;
  for (; take > 0; --take) {
    sel |= rest & (0u - rest);  // lowest remaining tie
    rest &= rest - 1u;
  }
  const int c = __popc(sel);
  int pos = warp_incl_scan(c, lane) - c;
  while (sel) {
    irow[pos++] = 32 * lane + (__ffs(sel) - 1);
    sel &= sel - 1u;
  }
}

// Ids of the Kt largest of the row's C keys (in shared memory, any Kt), ties
// to the lower id, ascending: the Kt-th largest key by the bit search over
// all keys, then the ids above it and the lowest-id ones equal to it.
__device__ __forceinline__ void topk_full_search(const uint32_t* keys, int C, int Kt, int lane, int32_t* irow) {
  const uint32_t lt_mask = (1u << lane) - 1u;
  const uint32_t T = kth_largest(keys, C, Kt, lane);
  unsigned gt = 0;
  for (int j = lane; j < C; j += 32) gt += (keys[j] > T);
  const int need = Kt - (int)__reduce_add_sync(0xffffffffu, gt);
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < C; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t k = j < C ? keys[j] : 0u;
    const bool is_eq = j < C && k == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take = (j < C && k > T) || (is_eq && eq_seen + __popc(eqb & lt_mask) < need);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) irow[pos + __popc(tb & lt_mask)] = j;
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

// Top-K for Kt <= 32 and C <= 1024 with the row in registers. The minimum of
// the lanes' maxima bounds the Kt-th largest key from below (every lane holds
// at least one key when C >= 64; below that a lane without keys contributes
// 0, so every key is a candidate). Each lane counts its keys at or above the
// bound, a prefix sum over the lanes places them, and they are written to
// shared memory with their ids before the exponentials overwrite the row; the
// selection then runs over the candidates alone. More than kCandCap
// candidates (e.g. many equal scores) fall back to all keys in shared memory
// and the full search.
__device__ __forceinline__ void select_topk_regs(const CoarseParams& p, int row, uint32_t* keys, int* cidx,
                                                 uint32_t* bm, int lane) {
  const int C = p.C, Kt = p.topk;
  float v[32];
  load_row_regs(p, row, lane, v);
  // The row as keys, in place (the key map is a bijection: key_value undoes it
  // exactly, -inf padding included), so only one copy of the row is live.
  uint32_t lkmax = 0;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const uint32_t k = order_key(v[e]);
    v[e] = __uint_as_float(k);
    if (64 * (e >> 1) + 2 * lane + (e & 1) < C) lkmax = max(lkmax, k);
  }
  const uint32_t lo = __reduce_min_sync(0xffffffffu, lkmax);
  const uint32_t hi = __reduce_max_sync(0xffffffffu, lkmax);
  int nl = 0;
#pragma unroll
  for (int e = 0; e < 32; ++e)
    nl += (64 * (e >> 1) + 2 * lane + (e & 1) < C && __float_as_uint(v[e]) >= lo) ? 1 : 0;
  const int incl = warp_incl_scan(nl, lane);
  const int n = __shfl_sync(0xffffffffu, incl, 31);
  if (n <= kCandCap) {
    int pos = incl - nl;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = 64 * (e >> 1) + 2 * lane + (e & 1);
      const uint32_t k = __float_as_uint(v[e]);
      if (j < C && k >= lo) {
        keys[pos] = k;
        cidx[pos] = j;
        ++pos;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = 64 * (e >> 1) + 2 * lane + (e & 1);
      if (j < C) keys[j] = __float_as_uint(v[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = key_value(__float_as_uint(v[e]));
  float mb, l;
  softmax_store_regs<true>(p, row, lane, v, key_value(hi), mb, l);
  __syncwarp();
  int32_t* irow = p.idx + (size_t)row * p.kcap;
  if (n <= 32) topk_bitmap_emit<1>(keys, cidx, n, Kt, lo, hi, bm, irow);
  else if (n <= 64) topk_bitmap_emit<2>(keys, cidx, n, Kt, lo, hi, bm, irow);
  else if (n <= 128) topk_bitmap_emit<4>(keys, cidx, n, Kt, lo, hi, bm, irow);
  else if (n <= kCandCap) topk_bitmap_emit<8>(keys, cidx, n, Kt, lo, hi, bm, irow);
  else topk_full_search(keys, C, Kt, lane, irow);
  if (lane == 0) p.cnt[row] = Kt;
}

// Fixed top-K (any K), and the probabilities alone when the selection is
// supplied by the caller, with the row's keys in shared memory instead of
// registers, so more warps (rows) per SM hide the latency of the warp-wide
// reductions. One warp per row; per warp the shared memory holds the keys
// (C rounded up to 32) and kCandCap candidate ids. Passes: load the scores as
// keys (lane maxima of score and key), the row sum, the probabilities as three
// bf16 terms, then the selection. For K <= 32 the minimum of the lanes'
// maxima bounds the K-th largest key from below, and the search runs over the
// candidates at or above it, compacted in place; larger K, or more than
// kCandCap candidates, take the bit search over all keys.
template <bool REGS>
__global__ void __launch_bounds__(256, 4) coarse_select_topk_kernel(const CoarseParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= p.BH * p.C) return;
  const int C = p.C, Kt = p.topk;
  const int stride = (C + 31) / 32 * 32;
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn) + (size_t)warp * (stride + kCandCap + 64);
  int* cidx = reinterpret_cast<int*>(keys + stride);
  const uint32_t lt_mask = (1u << lane) - 1u;
  float mb, l;
  uint32_t lkmax;
  if (REGS) row_softmax_regs(p, row, keys, lane, mb, l, lkmax);
  else row_softmax(p, row, keys, lane, mb, l, lkmax);
  if (!p.do_select) return;
  int32_t* irow = p.idx + (size_t)row * p.kcap;
  // Lower bound lo of the Kt-th largest key (for Kt <= 32: every lane with a
  // key holds one at or above it) and the row maximum hi.
  const uint32_t lo = __reduce_min_sync(0xffffffffu, lane < C ? lkmax : 0xffffffffu);
  const uint32_t hi = __reduce_max_sync(0xffffffffu, lkmax);
  int n = kCandCap + 1;
  if (Kt <= 32) {
    unsigned nl = 0;
    for (int j = lane; j < C; j += 32) nl += (keys[j] >= lo);
    n = (int)__reduce_add_sync(0xffffffffu, nl);
  }
  if (n <= kCandCap) {
    // In-place compaction in ascending id order: a candidate never lands past
    // the position it is read from, and every lane reads before the ballot.
    int pos = 0;
    for (int j0 = 0; j0 < C; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t k = j < C ? keys[j] : 0u;
      const bool t = j < C && k >= lo;
      const unsigned tb = __ballot_sync(0xffffffffu, t);
      if (t) {
        const int q = pos + __popc(tb & lt_mask);
        keys[q] = k;
        cidx[q] = j;
      }
      pos += __popc(tb);
    }
    __syncwarp();
    if (n <= 32) topk_from_candidates<1>(keys, cidx, n, Kt, lo, hi, irow);
    else if (n <= 64) topk_from_candidates<2>(keys, cidx, n, Kt, lo, hi, irow);
    else if (n <= 128) topk_from_candidates<4>(keys, cidx, n, Kt, lo, hi, irow);
    else topk_from_candidates<8>(keys, cidx, n, Kt, lo, hi, irow);
  } else {
    topk_full_search(keys, C, Kt, lane, irow);
  }
  if (lane == 0) p.cnt[row] = Kt;
}

// Top-K for Kt <= 32 and C <= 1024 (select_topk_regs), one warp per row;
// per warp the shared memory holds the candidates' keys (C rounded up to 32),
// kCandCap candidate ids and the two emission bitmaps.
__global__ void __launch_bounds__(256, 3) coarse_select_topk_regs_kernel(const CoarseParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= p.BH * p.C) return;
  const int stride = (p.C + 31) / 32 * 32;
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn) + (size_t)warp * (stride + kCandCap + 64);
  int* cidx = reinterpret_cast<int*>(keys + stride);
  select_topk_regs(p, row, keys, cidx, reinterpret_cast<uint32_t*>(cidx + kCandCap), lane);
}

// Top-p selection with the row's keys in shared memory: the kmax best
// candidates (the exact kmax-th largest key by the bit search, ties to the
// lower id) are ranked by score and cut at the first prefix whose probability
// mass reaches top_p * l, clamped to [kmin, kmax]; the ids go out ascending.
// One warp per row; per warp the shared memory holds the keys (C rounded up
// to 32) and four kmax-entry arrays: candidate id (with its rank packed above
// it), key, weight, and the weights in rank order. Warps per CTA: blockDim / 32.
__global__ void __launch_bounds__(256, 2) coarse_select_topp_kernel(const CoarseParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= p.BH * p.C) return;
  const int C = p.C, Kt = p.kmax;
  const int stride = (C + 31) / 32 * 32;
  uint32_t* keys = reinterpret_cast<uint32_t*>(dyn) + (size_t)warp * (stride + 4 * Kt);
  int* cid = reinterpret_cast<int*>(keys + stride);
  uint32_t* ckey = keys + stride + Kt;
  float* cw = reinterpret_cast<float*>(keys + stride + 2 * Kt);
  float* sorted = reinterpret_cast<float*>(keys + stride + 3 * Kt);
  const uint32_t lt_mask = (1u << lane) - 1u;
  float mb, l;
  uint32_t lkmax;
  row_softmax(p, row, keys, lane, mb, l, lkmax);
  int32_t* irow = p.idx + (size_t)row * p.kcap;

  // The Kt candidates: keys above the Kt-th largest T and the lowest-id ones
  // equal to it, in ascending id order, with their softmax numerators.
  const uint32_t T = kth_largest(keys, C, Kt, lane);
  unsigned gtl = 0;
  for (int j = lane; j < C; j += 32) gtl += (keys[j] > T);
  const int need = Kt - (int)__reduce_add_sync(0xffffffffu, gtl);
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < C; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t k = j < C ? keys[j] : 0u;
    const bool is_eq = j < C && k == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take = (j < C && k > T) || (is_eq && eq_seen + __popc(eqb & lt_mask) < need);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int q = pos + __popc(tb & lt_mask);
      cid[q] = j;
      ckey[q] = k;
      cw[q] = fast_exp2(fmaf(key_value(k), kLog2e, -mb));
    }
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
  __syncwarp();
  // Rank = number of candidates ahead in (score desc, id asc) order.
  for (int c = lane; c < Kt; c += 32) {
    const uint32_t kc = ckey[c];
    int r = 0;
    for (int o = 0; o < Kt; ++o) {
      const uint32_t ko = ckey[o];
      r += (ko > kc) || (ko == kc && o < c);  // candidates are stored in ascending id
    }
    sorted[r] = cw[c];
    cid[c] = cid[c] | (r << 16);  // pack rank above the id (ids < 65536)
  }
  __syncwarp();
  // First rank whose cumulative weight reaches top_p * l.
  const int CH = (Kt + 31) / 32;
  const int b0 = lane * CH, b1 = min(b0 + CH, Kt);
  float part = 0.f;
  for (int r = b0; r < b1; ++r) part += sorted[r];
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
    run += sorted[r];
    if (run >= target) {
      first = r;
      break;
    }
  }
  first = __reduce_min_sync(0xffffffffu, first);
  int nsel = (first == 0x7fffffff) ? Kt : first + 1;
  nsel = max(nsel, p.kmin);
  nsel = min(nsel, Kt);
  // Candidates with rank < nsel, in ascending id order.
  int opos = 0;
  for (int c0 = 0; c0 < Kt; c0 += 32) {
    const int c = c0 + lane;
    const int packed = (c < Kt) ? cid[c] : 0;
    const bool take = (c < Kt) && ((packed >> 16) < nsel);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) irow[opos + __popc(tb & lt_mask)] = packed & 0xffff;
    opos += __popc(tb);
  }
  for (int c = nsel + lane; c < p.kcap; c += 32) irow[c] = -1;
  if (lane == 0) p.cnt[row] = nsel;
}

// ------------------------------------------------------------ 1 / 3. three-term bf16 GEMM
// One CTA per 128-row tile: warp 0 issues the TMA loads (all three terms of A
// and B for 64 columns of K per stage; one stage for the scores, two for the
// output), warp 1 the 6 x 4 MMAs of
// a stage (M=128, K=16 each), and all four warps read the fp32 accumulator
// out of tensor memory.
//   KIND 0 (scores): A = qbar terms [C x D], B = kbar terms [C x D] (both
//          K-major), N tile 128 key cubes, K = D; out = S * scale.
//   KIND 1 (output): A = P terms [C x Cp] (K-major), B = vbar terms [C x D]
//          (N-major), N = D, K = Cp; out = Oc (and the optional copy).
// Every wait is bounded; a wait that gives up records kErrTimeout.
template <int KIND, int D>
struct TcShape {
  // Bf16 terms used per operand and products summed: the scores decide
  // integer selections and keep all three terms (six products, dropped terms
  // below 2^-24 relative). The coarse output decides nothing and is checked
  // against the fp64 oracle at 1e-4: hi + mid (16 significant bits, error
  // <= 2^-18 relative) and the products hi.hi, hi.mid, mid.hi leave an error
  // of a few 2^-18 relative, about 2e-5 absolute for these means.
  static constexpr int TERMS = KIND == 0 ? 3 : 2;
  static constexpr int PRODUCTS = KIND == 0 ? 6 : 3;
  static constexpr int NT = KIND == 0 ? 128 : D;    // accumulator columns
  static constexpr int A_BYTES = 128 * 64 * 2;      // one term, 128 rows x 64 K
  static constexpr int B_BYTES = NT * 64 * 2;       // one term
  static constexpr int STAGE = TERMS * (A_BYTES + B_BYTES);
  // Scores: K = D is one or two 64-column chunks, so a single stage lets two
  // CTAs share an SM and overlap each other's loads, MMAs and epilogue.
  // Output: K = Cp is up to 64 chunks, double-buffered.
  static constexpr int NS = KIND == 0 ? 1 : 2;
  static constexpr int SMEM = NS * STAGE + 1024;
};

template <int KIND, int D>
__global__ void __launch_bounds__(128, KIND == 0 ? 2 : 1) coarse_tc_kernel(const __grid_constant__ CoarseParams p) {
  using S = TcShape<KIND, D>;
  using namespace ptx;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[2], empty[2], done;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C, BH = p.BH;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * S::NT, bh = blockIdx.z;
  const int K = KIND == 0 ? D : p.Cp;
  const int nch = (K + 63) / 64;
  const uint64_t lim = p.wait_ns;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  auto a_tile = [&](int st, int t) { return tiles + st * S::STAGE + t * S::A_BYTES; };
  auto b_tile = [&](int st, int t) { return tiles + st * S::STAGE + S::TERMS * S::A_BYTES + t * S::B_BYTES; };

  if (warp == 0 && lane == 0) {
    const CUtensorMap* ta = KIND == 0 ? &p.tm_qs : &p.tm_ps;
    const CUtensorMap* tb = KIND == 0 ? &p.tm_ks : &p.tm_vs;
    int armed = 0;
    for (int c = 0; c < nch; ++c) {
      const int st = c % S::NS;
      if (c >= S::NS && !mbar_wait(&empty[st], ((c / S::NS) - 1) & 1, lim)) {
        atomicOr(p.err, kErrTimeout);
        break;
      }
      mbar_arrive_expect_tx(&full[st], S::STAGE);
      ++armed;
      for (int t = 0; t < S::TERMS; ++t) {
        tma_load_3d(a_tile(st, t), ta, &full[st], 64 * c, m0, t * BH + bh);
        if (KIND == 0) {
          tma_load_3d(b_tile(st, t), tb, &full[st], 64 * c, n0, t * BH + bh);
        } else {
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_load_3d(b_tile(st, t) + h * 8192, tb, &full[st], 64 * h, 64 * c, t * BH + bh);
        }
      }
    }
    // Drain: the last armed phase of each stage covers all copies issued.
    for (int st = 0; st < S::NS && st < armed; ++st) mbar_wait(&full[st], ((armed - 1 - st) / S::NS) & 1, lim);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, S::NT, false, KIND == 1);
    // Term pairs (A term, B term) of the six products kept.
    // term pairs, smallest products first: all six pairs above 2^-24 (scores),
    // or mid.hi, hi.mid, hi.hi (output)
    constexpr int pa[6] = {KIND == 0 ? 2 : 1, 0, 1, 1, 0, 0}, pb[6] = {0, KIND == 0 ? 2 : 1, 1, 0, 1, 0};
    constexpr int q0 = 6 - S::PRODUCTS;
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int st = c % S::NS;
      if (!mbar_wait(&full[st], (c / S::NS) & 1, lim)) {
        atomicOr(p.err, kErrTimeout);
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int q = q0; q < 6; ++q) {
          const uint64_t ad = sdesc_sw128(smem_u32(a_tile(st, pa[q])), 16, 1024) + (uint64_t)((kk * 32) >> 4);
          uint64_t bd;
          if (KIND == 0) bd = sdesc_sw128(smem_u32(b_tile(st, pb[q])), 16, 1024) + (uint64_t)((kk * 32) >> 4);
          else bd = sdesc_sw128(smem_u32(b_tile(st, pb[q])), 8192, 1024) + (uint64_t)((kk * 2048) >> 4);
          mma_bf16_ss(tmem, ad, bd, idesc, (c > 0 || kk > 0 || q > q0) ? 1u : 0u);
        }
      mma_commit(&empty[st]);
    }
    mma_commit(&done);
  }
  __syncwarp();
  // Epilogue: warp w holds accumulator rows 32 w .. 32 w + 31 (one per thread).
  const bool have = __all_sync(0xffffffffu, mbar_wait(&done, 0, lim));  // warp-uniform: the staged path syncs the warp
  if (!have && lane == 0) atomicOr(p.err, kErrTimeout);
  tc_fence_after();
  const int row = m0 + 32 * warp + lane;
  // Scores: each 32-column group goes through a per-warp [32 rows][36 floats]
  // staging block in the (now idle) operand stage, so that every warp store
  // writes four whole 128-byte row segments instead of 16 bytes in each of 32
  // rows. float4 writes and reads both touch 8 distinct bank groups per
  // quarter warp (row pitch 9 chunks of 16 bytes).
  float* stg = reinterpret_cast<float*>(tiles) + warp * 32 * 36;
  const bool staged = KIND == 0 && (C & 3) == 0;
#pragma unroll
  for (int cg = 0; cg < S::NT / 32; ++cg) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * cg, r);
    tmem_wait_ld();
    if (KIND == 0 && staged) {
      if (!have) continue;
      __syncwarp();  // the previous group's reads of the block are done
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(stg + lane * 36 + e) =
            make_float4(__uint_as_float(r[e]) * p.scale, __uint_as_float(r[e + 1]) * p.scale,
                        __uint_as_float(r[e + 2]) * p.scale, __uint_as_float(r[e + 3]) * p.scale);
      __syncwarp();
      const int col = n0 + 32 * cg + 4 * (lane & 7);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 4 * i + (lane >> 3), grow = m0 + 32 * warp + rr;
        if (grow < C && col < C)  // C % 4 == 0: a chunk lies wholly inside or outside the row
          *reinterpret_cast<float4*>(p.s + ((size_t)bh * C + grow) * C + col) =
              *reinterpret_cast<const float4*>(stg + rr * 36 + 4 * (lane & 7));
      }
      continue;
    }
    if (!have || row >= C) continue;
    if (KIND == 0) {
      float* dst = p.s + ((size_t)bh * C + row) * C + n0 + 32 * cg;
      const int ncol = min(32, C - (n0 + 32 * cg));
      {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < ncol) dst[e] = __uint_as_float(r[e]) * p.scale;
      }
    } else {
      const size_t o = ((size_t)bh * C + row) * D + 32 * cg;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 v = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                     __uint_as_float(r[e + 3]));
        *reinterpret_cast<float4*>(p.oc + o + e) = v;
        if (p.oc_copy) *reinterpret_cast<float4*>(p.oc_copy + o + e) = v;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int KIND, int D>
cudaError_t launch_tc(const CoarseParams& p, cudaStream_t st) {
  using S = TcShape<KIND, D>;
  cudaError_t e = cudaFuncSetAttribute(coarse_tc_kernel<KIND, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.C + 127) / 128, KIND == 0 ? (p.C + 127) / 128 : 1, p.BH);
  coarse_tc_kernel<KIND, D><<<grid, 128, S::SMEM, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_select_topk(const CoarseParams& p, cudaStream_t st) {
  const int rows = p.BH * p.C;
  const size_t smem = (size_t)8 * ((p.C + 31) / 32 * 32 + kCandCap + 64) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = p.C <= 1024 ? cudaFuncSetAttribute(coarse_select_topk_kernel<true>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                                : cudaFuncSetAttribute(coarse_select_topk_kernel<false>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (p.C <= 1024 && p.topk <= 32 && p.do_select) {
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(coarse_select_topk_regs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    coarse_select_topk_regs_kernel<<<(rows + 7) / 8, 256, smem, st>>>(p);
  } else if (p.C <= 1024)
    coarse_select_topk_kernel<true><<<(rows + 7) / 8, 256, smem, st>>>(p);
  else
    coarse_select_topk_kernel<false><<<(rows + 7) / 8, 256, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_select_topp(const CoarseParams& p, cudaStream_t st) {
  const int rows = p.BH * p.C;
  const size_t per_warp = ((size_t)(p.C + 31) / 32 * 32 + 4 * (size_t)p.kmax) * 4;
  int wpc = 8;  // warps (rows) per CTA, as many as fit in 227 KB of shared memory
  while (wpc > 1 && per_warp * wpc > 227 * 1024) --wpc;
  const size_t smem = per_warp * wpc;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(coarse_select_topp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  coarse_select_topp_kernel<<<(rows + wpc - 1) / wpc, 32 * wpc, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_coarse(const CoarseParams& p, cudaStream_t st) {
  cudaError_t e = p.D == 128 ? launch_tc<0, 128>(p, st) : launch_tc<0, 64>(p, st);
  if (e != cudaSuccess) return e;
  e = (p.topk > 0 || !p.do_select) ? launch_select_topk(p, st) : launch_select_topp(p, st);
  if (e != cudaSuccess) return e;
  return p.D == 128 ? launch_tc<1, 128>(p, st) : launch_tc<1, 64>(p, st);
}

}  // namespace vsa
