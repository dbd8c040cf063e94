// Backward pass: per-token preparation, the coarse attention's backward, and
// the transposed selection lists.
//
// "Faster Video Diffusion with Trainable Sparse Attention", "Approach": the
// whole hierarchy (coarse stage, selection, fine stage, gated combine) is
// trained end to end as one differentiable kernel; "VSA: Faster Video
// Diffusion with Trainable Sparse Attention", "Abstract (arXiv)": a single
// differentiable kernel. The pages give no gradient formulas; these are the
// chain rule of the forward pass with the selection held fixed (an index
// choice has no gradient):
//   out_n = gc_n Oc[c(n)] + gf_n Of_n
//   dgc_n = dout_n . Oc[c(n)],  dgf_n = dout_n . Of_n
//   dOf_n = gf_n dout_n,        dOc[c] = sum over the cube's tokens of gc_n dout_n
//   fine:   delta_n = dOf_n . Of_n; P = exp(s - lse); dS = P (dOf V^T - delta)
//   coarse: delta_c = dOc . Oc; dSc = Pc (dOc vbar^T - delta_c);
//           dqbar = dSc kbar / sqrt(D), dkbar = dSc^T qbar / sqrt(D), dvbar = Pc^T dOc
//           (tensor cores, fp32-accurate three-term bf16 operands)
//   pool:   every token of cube c receives 1/64 of the pooled gradient.
#include "sm100_ptx.cuh"
#include "vsa_common.cuh"

namespace vsa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ prep
// One warp per query cube: D/8 lanes cover a token row (16 bytes each), a
// warp step covers 32/(D/8) rows. Writes gate_f * dout cube-major (the dO
// operand of the fine backward), the per-token statistics the fine kernels
// need (lse in log2 units, delta), the gate gradients, and the cube's dOc and
// delta_c.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const PrepParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPS = 32 / LPR;
  constexpr int STEPS = kCube / RPS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (c >= p.C) return;
  const int sub = lane / LPR, chunk = lane % LPR;
  const size_t cube = (size_t)bh * p.C + c;
  float oc[8], acc[8];
  {
    const float4* o4 = reinterpret_cast<const float4*>(p.oc + cube * D + chunk * 8);
    const float4 a = o4[0], b = o4[1];
    oc[0] = a.x; oc[1] = a.y; oc[2] = a.z; oc[3] = a.w; oc[4] = b.x; oc[5] = b.y; oc[6] = b.z; oc[7] = b.w;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float* st = p.qstat + cube * 128;
#pragma unroll 4
  for (int s = 0; s < STEPS; ++s) {
    const int r = s * RPS + sub;
    const int n = cube_token(c, r, p.H, p.W);
    const size_t row = (size_t)bh * p.N + n;
    const int4 dv = __ldg(reinterpret_cast<const int4*>(p.dout + row * D + chunk * 8));
    const float4 o_lo = __ldg(reinterpret_cast<const float4*>(p.ofine + row * D + chunk * 8));
    const float4 o_hi = __ldg(reinterpret_cast<const float4*>(p.ofine + row * D + chunk * 8 + 4));
    const float of[8] = {o_lo.x, o_lo.y, o_lo.z, o_lo.w, o_hi.x, o_hi.y, o_hi.z, o_hi.w};
    const float gc = __ldg(p.gate_c + row), gf = __ldg(p.gate_f + row);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
    // pc = dout . Oc (dgate_c), pf = dout . Of (dgate_f), pd = bf16(gf dout) . Of: delta,
    // formed from the same rounded dO the fine kernels' dP product uses, so that
    // sum_m P_m (dP_m - delta) stays close to zero (it multiplies the
    // P-weighted mean of the keys in dq).
    float pc = 0.f, pf = 0.f, pd = 0.f;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 d = __bfloat1622float2(d2[e]);
      pc = fmaf(d.x, oc[2 * e], fmaf(d.y, oc[2 * e + 1], pc));
      pf = fmaf(d.x, of[2 * e], fmaf(d.y, of[2 * e + 1], pf));
      acc[2 * e] = fmaf(gc, d.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(gc, d.y, acc[2 * e + 1]);
      const __nv_bfloat162 g = __floats2bfloat162_rn(gf * d.x, gf * d.y);
      const float2 gr = __bfloat1622float2(g);
      pd = fmaf(gr.x, of[2 * e], fmaf(gr.y, of[2 * e + 1], pd));
      w[e] = *reinterpret_cast<const uint32_t*>(&g);
    }
    *reinterpret_cast<uint4*>(p.do_cube + (cube * kCube + r) * D + chunk * 8) = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1) {
      pc += __shfl_xor_sync(0xffffffffu, pc, off);
      pf += __shfl_xor_sync(0xffffffffu, pf, off);
      pd += __shfl_xor_sync(0xffffffffu, pd, off);
    }
    if (chunk == 0) {
      p.dgate_c[row] = pc;
      p.dgate_f[row] = pf;
      st[r] = __ldg(p.lse + row) * kLog2e;
      st[64 + r] = pd;
    }
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  float dl = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) dl = fmaf(acc[e], oc[e], dl);
#pragma unroll
  for (int off = 1; off < LPR; off <<= 1) dl += __shfl_xor_sync(0xffffffffu, dl, off);
  if (sub == 0) {
    float4* d4 = reinterpret_cast<float4*>(p.doc + cube * D + chunk * 8);
    d4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    d4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    if (chunk == 0) p.dlc[cube] = dl;
    // dOc as three bf16 terms for the tensor-core coarse backward
    uint32_t w[3][4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float x[2] = {acc[e], acc[e + 1]};
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[0], x[1]);
        const float2 back = __bfloat1622float2(h);
        x[0] -= back.x;
        x[1] -= back.y;
        w[t][e / 2] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    const size_t plane = (size_t)p.BH * p.C * D;
#pragma unroll
    for (int t = 0; t < 3; ++t)
      *reinterpret_cast<uint4*>(p.docsplit + t * plane + cube * D + chunk * 8) = make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
  }
}

// ------------------------------------------------------------ coarse backward
// Four products per head on the tensor cores (tcgen05, M = 128, fp32 in TMEM),
// every fp32 operand as three bf16 terms x = hi + mid + lo and the six
// products hi.hi, hi.mid, mid.hi, mid.mid, hi.lo, lo.hi summed (the dropped
// ones are below 2^-24 relative), so the products keep fp32 accuracy: dS
// feeds sums that cancel (sum_j dS_ij = 0), like the fine path's.
//   KIND 0: dPc = dOc vbar^T   [C x C], K = D; epilogue dS = Pc (dPc - delta_c) as three terms
//   KIND 1: dqbar = dS kbar / sqrt(D)    [C x D], K = C (A = dS, K-major)
//   KIND 2: dkbar = dS^T qbar / sqrt(D)  [C x D], K = C (A = dS^T, MN-major loads of dS)
//   KIND 3: dvbar = Pc^T dOc             [C x D], K = C (A = Pc^T, MN-major loads of Pc)
// One CTA per 128-row tile: warp 0 issues the TMA loads (all three terms of
// A and B for 64 of K per stage), warp 1 the 6 x 4 MMAs of a stage, all four
// warps read the accumulator. Every wait is bounded (records kErrTimeout).
template <int KIND, int D>
struct BwTc {
  static constexpr int NT = KIND == 0 ? 128 : D;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = NT * 64 * 2;
  static constexpr int STAGE = 3 * (A_BYTES + B_BYTES);
  static constexpr int NS = KIND == 0 ? 1 : 2;
  static constexpr int SMEM = NS * STAGE + 1024;
};

__device__ __forceinline__ void split3(float x, __nv_bfloat16& h, __nv_bfloat16& m, __nv_bfloat16& l) {
  h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  m = __float2bfloat16_rn(r1);
  l = __float2bfloat16_rn(r1 - __bfloat162float(m));
}

template <int KIND, int D>
__global__ void __launch_bounds__(128, KIND == 0 ? 2 : 1)
    coarse_bwd_tc_kernel(const __grid_constant__ CoarseBwdParams p) {
  using S = BwTc<KIND, D>;
  using namespace ptx;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[2], empty[2], done;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C, BH = p.BH;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * S::NT, bh = blockIdx.z;
  const int K = KIND == 0 ? D : (KIND == 1 ? p.Cp : C);
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
    tmem_alloc(&tmem_base, S::NT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  auto a_tile = [&](int st, int t) { return tiles + st * S::STAGE + t * S::A_BYTES; };
  auto b_tile = [&](int st, int t) { return tiles + st * S::STAGE + 3 * S::A_BYTES + t * S::B_BYTES; };

  if (warp == 0 && lane == 0) {
    int armed = 0;
    for (int c = 0; c < nch; ++c) {
      const int st = c % S::NS;
      if (c >= S::NS && !mbar_wait(&empty[st], ((c / S::NS) - 1) & 1, lim)) {
        atomicOr(p.err, kErrTimeout);
        break;
      }
      mbar_arrive_expect_tx(&full[st], S::STAGE);
      ++armed;
      for (int t = 0; t < 3; ++t) {
        const int plane = t * BH + bh;
        if (KIND == 0) {
          tma_load_3d(a_tile(st, t), &p.tm_doc128, &full[st], 64 * c, m0, plane);
          tma_load_3d(b_tile(st, t), &p.tm_vb128, &full[st], 64 * c, n0, plane);
        } else {
          if (KIND == 1) {
            tma_load_3d(a_tile(st, t), &p.tm_ds128, &full[st], 64 * c, m0, plane);
          } else {
            const CUtensorMap* ta = KIND == 2 ? &p.tm_ds64 : &p.tm_p64;
#pragma unroll
            for (int mh = 0; mh < 2; ++mh) tma_load_3d(a_tile(st, t) + mh * 8192, ta, &full[st], m0 + 64 * mh, 64 * c, plane);
          }
          const CUtensorMap* tb = KIND == 1 ? &p.tm_kb64 : (KIND == 2 ? &p.tm_qb64 : &p.tm_doc64);
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_load_3d(b_tile(st, t) + h * 8192, tb, &full[st], 64 * h, 64 * c, plane);
        }
      }
    }
    for (int st = 0; st < S::NS && st < armed; ++st) mbar_wait(&full[st], ((armed - 1 - st) / S::NS) & 1, lim);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, S::NT, KIND >= 2, KIND >= 1);
    constexpr int pa[6] = {2, 0, 1, 1, 0, 0}, pb[6] = {0, 2, 1, 0, 1, 0};
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
        for (int q = 0; q < 6; ++q) {
          uint64_t ad, bd;
          if (KIND >= 2) ad = sdesc_sw128(smem_u32(a_tile(st, pa[q])), 8192, 1024) + (uint64_t)((kk * 2048) >> 4);
          else ad = sdesc_sw128(smem_u32(a_tile(st, pa[q])), 16, 1024) + (uint64_t)((kk * 32) >> 4);
          if (KIND == 0) bd = sdesc_sw128(smem_u32(b_tile(st, pb[q])), 16, 1024) + (uint64_t)((kk * 32) >> 4);
          else bd = sdesc_sw128(smem_u32(b_tile(st, pb[q])), 8192, 1024) + (uint64_t)((kk * 2048) >> 4);
          mma_bf16_ss(tmem, ad, bd, idesc, (c > 0 || kk > 0 || q > 0) ? 1u : 0u);
        }
      mma_commit(&empty[st]);
    }
    mma_commit(&done);
  }
  __syncwarp();
  const bool have = mbar_wait(&done, 0, lim);
  if (!have && lane == 0) atomicOr(p.err, kErrTimeout);
  tc_fence_after();
  const int row = m0 + 32 * warp + lane;
  const size_t cp_plane = (size_t)BH * C * p.Cp;
#pragma unroll 1
  for (int cg = 0; cg < S::NT / 32; ++cg) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * cg, r);
    tmem_wait_ld();
    if (!have || row >= C) continue;
    if (KIND == 0) {
      const int j0 = n0 + 32 * cg;
      if (j0 >= p.Cp) continue;
      const float dl = p.dlc[(size_t)bh * C + row];
      const size_t o = ((size_t)bh * C + row) * p.Cp + j0;
      if (j0 + 32 <= C) {
        // 32 columns of the row: 16-byte loads of the three P terms and 16-byte
        // stores of the three dS terms (row pitch Cp * 2 bytes, a multiple of 16)
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 pt[3];
#pragma unroll
          for (int t = 0; t < 3; ++t) pt[t] = *reinterpret_cast<const uint4*>(p.psplit + t * cp_plane + o + 8 * v4);
          uint32_t w[3][4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float ds[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 8 * v4 + 2 * e2 + h2;
              float P = 0.f;
#pragma unroll
              for (int t = 0; t < 3; ++t) {
                const uint32_t word = (&pt[t].x)[e2];
                P += __uint_as_float((h2 ? (word & 0xffff0000u) : (word << 16)));
              }
              ds[h2] = P * (__uint_as_float(r[e]) - dl);
            }
            float x[2] = {ds[0], ds[1]};
#pragma unroll
            for (int t = 0; t < 3; ++t) {
              const __nv_bfloat162 hh = __floats2bfloat162_rn(x[0], x[1]);
              const float2 back = __bfloat1622float2(hh);
              x[0] -= back.x;
              x[1] -= back.y;
              w[t][e2] = *reinterpret_cast<const uint32_t*>(&hh);
            }
          }
#pragma unroll
          for (int t = 0; t < 3; ++t)
            *reinterpret_cast<uint4*>(p.dssplit + t * cp_plane + o + 8 * v4) = make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = j0 + e;
          if (j >= p.Cp) continue;
          float ds = 0.f;
          if (j < C) {
            const float P = __bfloat162float(p.psplit[o + e]) + __bfloat162float(p.psplit[cp_plane + o + e]) +
                            __bfloat162float(p.psplit[2 * cp_plane + o + e]);
            ds = P * (__uint_as_float(r[e]) - dl);
          }
          __nv_bfloat16 h, m, l;
          split3(ds, h, m, l);
          p.dssplit[o + e] = h;
          p.dssplit[cp_plane + o + e] = m;
          p.dssplit[2 * cp_plane + o + e] = l;
        }
      }
    } else {
      float* out = KIND == 1 ? p.dqbar : (KIND == 2 ? p.dkbar : p.dvbar);
      const float alpha = KIND == 3 ? 1.0f : p.scale;
      const size_t o = ((size_t)bh * C + row) * D + 32 * cg;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(out + o + e) =
            make_float4(alpha * __uint_as_float(r[e]), alpha * __uint_as_float(r[e + 1]),
                        alpha * __uint_as_float(r[e + 2]), alpha * __uint_as_float(r[e + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, S::NT);
  }
}

template <int KIND, int D>
cudaError_t launch_bw_tc(const CoarseBwdParams& p, cudaStream_t st) {
  using S = BwTc<KIND, D>;
  cudaError_t e =
      cudaFuncSetAttribute(coarse_bwd_tc_kernel<KIND, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.C + 127) / 128, KIND == 0 ? (p.Cp + 127) / 128 : 1, p.BH);
  coarse_bwd_tc_kernel<KIND, D><<<grid, 128, S::SMEM, st>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_coarse_bwd_t(const CoarseBwdParams& p, cudaStream_t st) {
  cudaError_t e = launch_bw_tc<0, D>(p, st);
  if (e == cudaSuccess) e = launch_bw_tc<1, D>(p, st);
  if (e == cudaSuccess) e = launch_bw_tc<2, D>(p, st);
  if (e == cudaSuccess) e = launch_bw_tc<3, D>(p, st);
  return e;
}

// ------------------------------------------------------------ transposed lists
// Marks bit (j, i) for every selected pair (query cube i, KV cube j). Ids
// outside [0, C), counts outside [1, kcap] and rows that are not strictly
// ascending are reported (kErrBadIndex) and skipped, never used as addresses.
__global__ void tlist_mark_kernel(const TlistParams p) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.BH * p.C * p.kcap;
  if (t >= total) return;
  const long long row = t / p.kcap;
  const int e = (int)(t - row * p.kcap);
  int n = p.cnt ? p.cnt[row] : p.kcap;
  if (n < 1 || n > p.kcap) {
    if (e == 0) atomicOr(p.err, kErrBadIndex);
    n = n < 1 ? 0 : p.kcap;
  }
  if (e >= n) return;
  const int j = p.idx[row * p.kcap + e];
  if (j < 0 || j >= p.C || (e > 0 && p.idx[row * p.kcap + e - 1] >= j)) {
    atomicOr(p.err, kErrBadIndex);
    return;
  }
  const int bh = (int)(row / p.C), i = (int)(row - (long long)bh * p.C);
  atomicOr(&p.bitmap[((size_t)bh * p.C + j) * p.W32 + (i >> 5)], 1u << (i & 31));
}

// One CTA per (batch, head): counts per KV cube (popcounts of its bitmap
// row), an exclusive scan over the head's KV cubes, then each KV cube's query
// cubes in ascending order (the bit order), so the lists are deterministic.
__global__ void __launch_bounds__(1024) tlist_build_kernel(const TlistParams p) {
  __shared__ int wsum[32];
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = p.C, W32 = p.W32;
  const int per = (C + 1023) / 1024;  // rows per thread (consecutive)
  const int r0 = tid * per;
  const uint32_t* bm = p.bitmap + (size_t)bh * C * W32;
  int mine = 0;
  for (int r = r0; r < r0 + per && r < C; ++r) {
    int c = 0;
    for (int w = 0; w < W32; ++w) c += __popc(bm[(size_t)r * W32 + w]);
    p.tcnt[(size_t)bh * C + r] = c;
    mine += c;
  }
  // block exclusive scan of `mine`
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;  // inclusive
  }
  __syncthreads();
  int off = incl - mine + (warp > 0 ? wsum[warp - 1] : 0);
  const size_t base = (size_t)bh * C * p.kcap;
  for (int r = r0; r < r0 + per && r < C; ++r) {
    p.toff[(size_t)bh * C + r] = (int)(base + off);
    int pos = 0;
    for (int w = 0; w < W32; ++w) {
      uint32_t bits = bm[(size_t)r * W32 + w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        p.tlist[base + off + pos] = 32 * w + b;
        ++pos;
      }
    }
    off += pos;
  }
}

}  // namespace

cudaError_t launch_bwd_prep(const PrepParams& p, int D, cudaStream_t st) {
  const dim3 grid((p.C + 7) / 8, p.BH);
  if (D == 128)
    bwd_prep_kernel<128><<<grid, 256, 0, st>>>(p);
  else
    bwd_prep_kernel<64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_coarse_bwd(const CoarseBwdParams& p, cudaStream_t st) {
  return p.D == 128 ? launch_coarse_bwd_t<128>(p, st) : launch_coarse_bwd_t<64>(p, st);
}

cudaError_t launch_tlists(const TlistParams& p, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(p.bitmap, 0, (size_t)p.BH * p.C * p.W32 * 4, st);
  if (e != cudaSuccess) return e;
  const long long total = (long long)p.BH * p.C * p.kcap;
  tlist_mark_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tlist_build_kernel<<<p.BH, 1024, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace vsa
