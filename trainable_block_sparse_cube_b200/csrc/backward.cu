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
//   pool:   every token of cube c receives 1/64 of the pooled gradient.
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
  }
}

// ------------------------------------------------------------ coarse backward
// fp32 SIMT products on 64 x 64 output tiles (16-deep k chunks in shared
// memory, 4 x 4 outputs per thread). The coarse stage is C x C per head, a few
// percent of the backward pass's work.
constexpr int kT = 64, kKc = 16;

// dSc = Pc (dOc vbar^T - delta_c); also writes Pc in fp32 for the dvbar product.
__global__ void __launch_bounds__(256) coarse_ds_kernel(const CoarseBwdParams p) {
  __shared__ float As[kKc][kT + 4], Bs[kKc][kT + 4];
  const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
  const int m0 = blockIdx.x * kT, n0 = blockIdx.y * kT, bh = blockIdx.z;
  const int C = p.C, D = p.D;
  const float* A = p.doc + (size_t)bh * C * D;    // [C][D]: A(m, k) = doc[m][k]
  const float* B = p.vbar + (size_t)bh * C * D;   // B(k, n) = vbar[n][k]
  float acc[4][4] = {};
  for (int k0 = 0; k0 < D; k0 += kKc) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + 256 * e;
      const int m = idx >> 4, kk = idx & 15;
      As[kk][m] = (m0 + m < C) ? A[(size_t)(m0 + m) * D + k0 + kk] : 0.f;
      Bs[kk][m] = (n0 + m < C) ? B[(size_t)(n0 + m) * D + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kKc; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][tm * 4 + i];
        b[i] = Bs[kk][tn * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const size_t plane = (size_t)p.BH * C * p.Cp;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm * 4 + i;
    if (m >= C) continue;
    const float dl = p.dlc[(size_t)bh * C + m];
    const __nv_bfloat16* prow = p.psplit + ((size_t)bh * C + m) * p.Cp;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n >= C) continue;
      const float P = __bfloat162float(prow[n]) + __bfloat162float(prow[plane + n]) +
                      __bfloat162float(prow[2 * plane + n]);
      const size_t o = ((size_t)bh * C + m) * C + n;
      p.p32[o] = P;
      p.ds[o] = P * (acc[i][j] - dl);
    }
  }
}

// out[m][d] = alpha * sum_k A(m, k) * B[k][d] with M = K = C and N = D:
//   z = 0: dvbar = Pc^T dOc             (A(m, k) = p32[k][m])
//   z = 1: dqbar = dSc kbar / sqrt(D)   (A(m, k) = ds[m][k])
//   z = 2: dkbar = dSc^T qbar / sqrt(D) (A(m, k) = ds[k][m])
__global__ void __launch_bounds__(256) coarse_grad_kernel(const CoarseBwdParams p) {
  __shared__ float As[kKc][kT + 4], Bs[kKc][kT + 4];
  const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
  const int m0 = blockIdx.x * kT, n0 = blockIdx.y * kT;
  const int which = blockIdx.z % 3, bh = blockIdx.z / 3;
  const int C = p.C, D = p.D;
  const size_t cc = (size_t)bh * C * C, cd = (size_t)bh * C * D;
  const float* A = which == 0 ? p.p32 + cc : p.ds + cc;
  const bool at = which != 1;
  const float* B = (which == 0 ? p.doc : which == 1 ? p.kbar : p.qbar) + cd;
  float* out = (which == 0 ? p.dvbar : which == 1 ? p.dqbar : p.dkbar) + cd;
  const float alpha = which == 0 ? 1.f : p.scale;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < C; k0 += kKc) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + 256 * e;
      if (at) {
        const int m = idx & 63, kk = idx >> 6;
        As[kk][m] = (m0 + m < C && k0 + kk < C) ? A[(size_t)(k0 + kk) * C + m0 + m] : 0.f;
      } else {
        const int m = idx >> 4, kk = idx & 15;
        As[kk][m] = (m0 + m < C && k0 + kk < C) ? A[(size_t)(m0 + m) * C + k0 + kk] : 0.f;
      }
      const int n = idx & 63, kk = idx >> 6;
      Bs[kk][n] = (k0 + kk < C && n0 + n < D) ? B[(size_t)(k0 + kk) * D + n0 + n] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kKc; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][tm * 4 + i];
        b[i] = Bs[kk][tn * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm * 4 + i;
    if (m >= C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n < D) out[(size_t)m * D + n] = alpha * acc[i][j];
    }
  }
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
  const int tc = (p.C + kT - 1) / kT;
  coarse_ds_kernel<<<dim3(tc, tc, p.BH), 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  coarse_grad_kernel<<<dim3(tc, (p.D + kT - 1) / kT, 3 * p.BH), 256, 0, st>>>(p);
  return cudaGetLastError();
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
