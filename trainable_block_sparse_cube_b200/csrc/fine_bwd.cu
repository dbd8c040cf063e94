// Block-sparse fine attention, backward pass (tcgen05 / TMEM / TMA).
//
// "Faster Video Diffusion with Trainable Sparse Attention", "Approach" and
// "VSA: Faster Video Diffusion with Trainable Sparse Attention", "Abstract
// (arXiv)": the block-sparse fine attention is part of one differentiable
// kernel trained end to end. With the selection fixed, the gradients of
// O = softmax(Q K^T / sqrt(D)) V over a query cube's selected tokens are
//   P  = exp2(S * log2(e)/sqrt(D) - lse2)   (lse2: the forward's log2 denominator)
//   dP = dO V^T,  dS = P o (dP - delta),  delta_n = dO_n . O_n
//   dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D),  dV = P^T dO
// summed, for K and V, over every query cube that selected the KV cube.
//
// Two kernels, no atomics (deterministic):
//   dQ kernel   one item = one query cube; steps of two of its selected KV
//               cubes (128 keys). S = Q K^T and dP = dO V^T (M=64, N=128,
//               SS), dS in TMEM as bf16, dQ += dS K (M=64, N=D, TS: dS from
//               TMEM, K as an MN-major B). The S and dP buffers are released
//               when read, dS has buffers of its own, so the S product of the
//               next step never waits for the dQ product of this one.
//   dK/dV kernel one item = one KV cube; steps over the query cubes that
//               selected it (transposed lists). S^T = K Q^T and dP^T = V dO^T
//               (M=64, N=64, SS), P^T and dS^T in TMEM as bf16,
//               dV += P^T dO and dK += dS^T Q (M=64, N=D, TS).
// Every product has 64 query or key rows as M (one cube = one tile), so the
// accumulators use the M=64 TMEM layout (16 lanes of each 32-lane quarter);
// the softmax-side warps read and write them with the 16-lane shapes.
//
// Elementwise warps. dQ kernel: all eight work on every step, warp w on the
// rows of lane quarter w % 4 and key half (w - 4) / 4; their packed bf16-pair
// columns (32 per warp) go to a dS buffer of their own. dK/dV kernel: two
// groups of four take alternate steps (group g: the steps j with j % 2 == g),
// so the TMEM round trips of two steps overlap; a warp handles all 64 columns
// of its lane quarter and writes its 32 packed columns over the first 32 fp32
// columns it has already read (no other warp reads that quarter of the
// buffer). The MMA that reads them takes its K = 16 slices at packed columns
// 8k.
//
// Warp roles (512 threads), both kernels:
//   warp 0      TMA producer (tiles and the per-query statistics)
//   warp 1      issuer of the S (or S^T) MMAs; allocates tensor memory
//   warp 2      issuer of the dP (or dP^T) MMAs
//   warp 3      issuer of the accumulating MMAs (dQ; or dV and dK)
//   warps 4-11  elementwise: P, dS (warp w: lane quarter w % 4, step parity (w-4)/4)
//   warps 12-15 epilogue: accumulators -> scale, add the coarse path's
//               gradient / 64, bf16, 5-D TMA store into the raster output
// Every mbarrier wait is bounded (the plan's wait limit); a wait that gives
// up records kErrTimeout, raises a CTA-wide abort flag, and the CTA drains
// its own copies and MMAs before it releases TMEM and exits.
#include "sm100_ptx.cuh"
#include "vsa_common.cuh"

namespace vsa {

namespace {

using namespace ptx;

constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 3, 128;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// Packed bf16 column of K = 16 slice k of a 64-column step (see the header).
__device__ __forceinline__ uint32_t packed_col(int k) { return 8u * k; }

// K-major operand slice k (16 elements along D) of a 64-row tile laid out as
// D/64 blocks of [64 rows][128 B] in the 128-byte swizzle: descriptor offset.
__device__ __forceinline__ uint64_t kmajor_off(int k) { return (uint64_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4); }

struct Waiter {
  int* abort_flag;
  int* err;
  uint64_t limit;
  __device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 64; ++i)
        if (mbar_try_wait(bar, parity)) return true;
      if (*(volatile int*)abort_flag) return false;
      if (globaltimer_ns() - t0 > limit) {
        *(volatile int*)abort_flag = 1;
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
  __device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) const { mbar_wait(bar, parity, limit); }
};

// The item at the CTA's position `is`, or -1 past the end: without an order
// array items blockIdx.x + is * gridDim.x; with one, the positions of a
// serpentine hand-out of the array (each head's items longest first,
// schedule.cu).
__device__ __forceinline__ int item_at(const BwdFineParams& p, int is) {
  const int G = gridDim.x, c = blockIdx.x;
  const int pos = is * G + ((p.order && (is & 1)) ? G - 1 - c : c);
  if (pos >= p.n_items) return -1;
  return p.order ? p.order[pos] : pos;
}

// One item's position: the item at position is; n steps.
struct Cur {
  int is, item, n, t;
  bool live, bad;
};

// dQ kernel: counts from cnt (or kcap), validated to [1, kcap].
__device__ __forceinline__ void dq_enter(const BwdFineParams& p, Cur& c) {
  c.live = c.item >= 0;
  int n = c.live ? (p.cnt ? p.cnt[c.item] : p.kcap) : 0;
  if (c.live && (n < 1 || n > p.kcap)) {
    c.bad = true;
    n = n < 1 ? 1 : p.kcap;
  }
  c.n = n;
  c.t = 0;
}
// dK/dV kernel: counts from the transposed lists, in [0, C].
__device__ __forceinline__ void dkv_enter(const BwdFineParams& p, Cur& c) {
  c.live = c.item >= 0;
  int n = c.live ? p.cnt[c.item] : 0;
  n = n < 0 ? 0 : (n > p.C ? p.C : n);
  c.n = n;
  c.t = 0;
}
template <bool DKV>
__device__ __forceinline__ void cur_init(const BwdFineParams& p, Cur& c) {
  c.is = 0;
  c.item = item_at(p, 0);
  c.bad = false;
  if (DKV) dkv_enter(p, c); else dq_enter(p, c);
}
// Next item (skipping nothing: items with n = 0 are visited with no steps).
template <bool DKV>
__device__ __forceinline__ void cur_next_item(const BwdFineParams& p, Cur& c) {
  c.is += 1;
  c.item = item_at(p, c.is);
  if (DKV) dkv_enter(p, c); else dq_enter(p, c);
}

// Output tile of one item: rows ra and ra+8 (16-lane layout) of the D-column
// accumulator at TMEM column col, times `scale`, plus the coarse-path row
// cp[d] / 64, as bf16 into the 128-byte-swizzled staging tile, then one 5-D
// TMA store per 64 channels into the raster output (est == 0 issues).
template <int D>
__device__ __forceinline__ void store_tile(const float* o, float scale, const float* cp, uint8_t* stage, int ra,
                                           int tq, int est, const CUtensorMap* tm, int ct, int ch, int cw, int bh) {
  const uint32_t sw = (uint32_t)(ra & 7);
#pragma unroll
  for (int jj = 0; jj < D / 8; ++jj) {
    const int d = 8 * jj + 2 * tq;
    const float c0 = cp[d] * (1.0f / 64.0f), c1 = cp[d + 1] * (1.0f / 64.0f);
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(fmaf(scale, o[4 * jj], c0), fmaf(scale, o[4 * jj + 1], c1));
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(fmaf(scale, o[4 * jj + 2], c0), fmaf(scale, o[4 * jj + 3], c1));
    uint8_t* blk = stage + (jj >> 3) * 8192 + ((((uint32_t)jj & 7u) ^ sw) << 4) + 4 * tq;
    *reinterpret_cast<__nv_bfloat162*>(blk + ra * 128) = h0;
    *reinterpret_cast<__nv_bfloat162*>(blk + (ra + 8) * 128) = h1;
  }
  fence_proxy_async_smem();
  epi_sync();
  if (est == 0) {
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tma_store_5d(tm, stage + h * 8192, 64 * h, 4 * cw, 4 * ch, 4 * ct, bh);
    bulk_commit();
  }
}

// Reads rows ra, ra+8 of a D-column M=64 accumulator into o (layout of
// tmem_ld16x256b_x8 per 64 columns).
template <int D>
__device__ __forceinline__ void load_acc(uint32_t taddr, float* o) {
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint32_t r[32];
    tmem_ld16x256b_x8(taddr + 64u * h, r);
    tmem_wait_ld();
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) o[32 * h + jj] = __uint_as_float(r[jj]);
  }
}

// Elementwise step of the softmax warps: s (scores) and g (dP) of rows a and
// a+8 for 64 columns (layout of tmem_ld16x256b_x8); lse2 and delta per row
// (dQ kernel: ROWSTAT) or per column (dK/dV kernel). Writes P (packed bf16
// pairs) to pk_p and dS to pk_s (layout of the 16x128b.x8 store).
template <bool ROWSTAT>
__device__ __forceinline__ void p_ds(const uint32_t (&s)[32], const uint32_t (&g)[32], float sl2, float l0, float l1,
                                     float d0, float d1, const float* lse_col, const float* dl_col, int c0,
                                     uint32_t (&pk_p)[16], uint32_t (&pk_s)[16]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float la0 = l0, la1 = l0, lb0 = l1, lb1 = l1, da0 = d0, da1 = d0, db0 = d1, db1 = d1;
    if (!ROWSTAT) {
      const int c = c0 + 8 * j;
      const float2 lc = *reinterpret_cast<const float2*>(lse_col + c);
      const float2 dc = *reinterpret_cast<const float2*>(dl_col + c);
      la0 = lb0 = lc.x;
      la1 = lb1 = lc.y;
      da0 = db0 = dc.x;
      da1 = db1 = dc.y;
    }
    const float p00 = ex2(fmaf(__uint_as_float(s[4 * j]), sl2, -la0));
    const float p01 = ex2(fmaf(__uint_as_float(s[4 * j + 1]), sl2, -la1));
    const float p10 = ex2(fmaf(__uint_as_float(s[4 * j + 2]), sl2, -lb0));
    const float p11 = ex2(fmaf(__uint_as_float(s[4 * j + 3]), sl2, -lb1));
    const __nv_bfloat162 hp0 = __floats2bfloat162_rn(p00, p01);
    const __nv_bfloat162 hp1 = __floats2bfloat162_rn(p10, p11);
    const __nv_bfloat162 hs0 =
        __floats2bfloat162_rn(p00 * (__uint_as_float(g[4 * j]) - da0), p01 * (__uint_as_float(g[4 * j + 1]) - da1));
    const __nv_bfloat162 hs1 = __floats2bfloat162_rn(p10 * (__uint_as_float(g[4 * j + 2]) - db0),
                                                     p11 * (__uint_as_float(g[4 * j + 3]) - db1));
    pk_p[2 * j] = *reinterpret_cast<const uint32_t*>(&hp0);
    pk_p[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&hp1);
    pk_s[2 * j] = *reinterpret_cast<const uint32_t*>(&hs0);
    pk_s[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&hs1);
  }
}

// ============================================================ dQ kernel
// Steps of two selected KV cubes (128 keys), as in the forward kernel: per
// step 8 S MMAs (M=64, N=128), 8 dP MMAs (M=64, N=128) and 8 dQ MMAs (M=64,
// N=D, K=16 keys each). An odd count loads the last cube twice; the
// elementwise warps zero the repeated half's dS.
template <int D>
struct DqL {
  static constexpr int NH = D / 64;
  static constexpr int TILE = 64 * D * 2;               // one cube
  static constexpr int PAIR = 2 * TILE;                 // one step's K or V (two cubes)
  static constexpr int KS = 2, VS = 2;
  static constexpr int OFF_Q = 0;                       // Q[2]
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;       // dO[2]
  static constexpr int OFF_K = OFF_DO + 2 * TILE;       // K ring (pairs)
  static constexpr int OFF_V = OFF_K + KS * PAIR;       // V ring (pairs)
  static constexpr int OFF_STAGE = OFF_V + VS * PAIR;   // output staging
  static constexpr int OFF_STAT = OFF_STAGE + TILE;     // statistics [2][128] fp32
  static constexpr int BYTES = OFF_STAT + 2 * 512;
  static constexpr int SMEM = BYTES + 1024;
};
// A pair tile holds, per 64-channel group h (at h * 2 * 8192), the first
// cube's 64 rows and then the second's, 128 B each in the 128-byte swizzle:
// one 128-row K-major operand (S, dP) or one 128-key MN-major operand (dQ).
//
// dQ kernel tensor memory: one fp32 S and one fp32 dP buffer (128 columns
// each), released as soon as the elementwise warps have read them; two bf16
// dS buffers (64 packed columns; step j uses j % 2), released by the dQ
// product; the dQ accumulator (D columns).
constexpr uint32_t kQS = 0, kQP = 128, kQdS = 256, kQAcc = 384;

struct __align__(8) DqBars {
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];  // rings of DqL<D>::KS / VS slots
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, dp_full, s_free, dp_free;
  uint64_t ds_full[2], ds_free[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain[3];
};

struct alignas(16) DqShared {
  DqBars bar;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float cpre[2][128];  // coarse-path gradient row of an item
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) fine_dq_kernel(const __grid_constant__ BwdFineParams p) {
  using L = DqL<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ DqShared sh;
  DqBars& B = sh.bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Waiter W{&sh.abort_flag, p.err, p.wait_ns};
  const int C = p.C;

  if (tid == 0) {
    for (int i = 0; i < L::KS; ++i) { mbar_init(&B.k_full[i], 1); mbar_init(&B.k_empty[i], 1); }
    for (int i = 0; i < L::VS; ++i) { mbar_init(&B.v_full[i], 1); mbar_init(&B.v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&B.q_full[i], 1); mbar_init(&B.q_empty[i], 2 + 8); }
    mbar_init(&B.s_full, 1);
    mbar_init(&B.dp_full, 1);
    mbar_init(&B.s_free, 8);
    mbar_init(&B.dp_free, 8);
    for (int d = 0; d < 2; ++d) {
      mbar_init(&B.ds_full[d], 8);
      mbar_init(&B.ds_free[d], 1);
    }
    mbar_init(&B.acc_full, 1);
    mbar_init(&B.acc_empty, 4);
    for (int i = 0; i < 3; ++i) mbar_init(&B.drain[i], 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_do);
    prefetch_tmap(&p.tm_out0);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    regs_dec<56>();
    if (lane == 0) {
      bool aborted = false, bad = false;
      int gk = 0, gq = 0;  // K/V steps armed, items armed
      Cur c;
      cur_init<false>(p, c);
      while (c.live && !aborted) {
        const int bh = c.item / C;
        // Q, dO and the statistics of the item -> buffer is & 1.
        const int qb = c.is & 1;
        if (c.is >= 2 && !W.wait(&B.q_empty[qb], ((c.is >> 1) - 1) & 1)) { aborted = true; break; }
        mbar_arrive_expect_tx(&B.q_full[qb], 2 * L::TILE + 512);
        for (int h = 0; h < L::NH; ++h) {
          tma_load_2d(tiles + L::OFF_Q + qb * L::TILE + h * 8192, &p.tm_q, &B.q_full[qb], 64 * h, c.item * 64);
          tma_load_2d(tiles + L::OFF_DO + qb * L::TILE + h * 8192, &p.tm_do, &B.q_full[qb], 64 * h, c.item * 64);
        }
        bulk_load(tiles + L::OFF_STAT + qb * 512, p.qstat + (size_t)c.item * 128, 512, &B.q_full[qb]);
        ++gq;
        const int steps = (c.n + 1) >> 1;
        for (int t = 0; t < steps; ++t) {
          int ja = p.list[(size_t)c.item * p.kcap + 2 * t];
          int jb = 2 * t + 1 < c.n ? p.list[(size_t)c.item * p.kcap + 2 * t + 1] : ja;  // odd tail: a copy
          if (ja < 0 || ja >= C) { bad = true; ja = 0; }
          if (jb < 0 || jb >= C) { bad = true; jb = 0; }
          const int ra = (bh * C + ja) * 64, rb = (bh * C + jb) * 64;
          const int ks = gk % L::KS, vs = gk % L::VS;
          if (gk >= L::KS && !W.wait(&B.k_empty[ks], ((gk / L::KS) - 1) & 1)) { aborted = true; break; }
          mbar_arrive_expect_tx(&B.k_full[ks], L::PAIR);
          uint8_t* kd = tiles + L::OFF_K + ks * L::PAIR;
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(kd + h * 16384, &p.tm_k, &B.k_full[ks], 64 * h, ra);
            tma_load_2d(kd + h * 16384 + 8192, &p.tm_k, &B.k_full[ks], 64 * h, rb);
          }
          if (gk >= L::VS && !W.wait(&B.v_empty[vs], ((gk / L::VS) - 1) & 1)) { aborted = true; break; }
          mbar_arrive_expect_tx(&B.v_full[vs], L::PAIR);
          uint8_t* vd = tiles + L::OFF_V + vs * L::PAIR;
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(vd + h * 16384, &p.tm_v, &B.v_full[vs], 64 * h, ra);
            tma_load_2d(vd + h * 16384 + 8192, &p.tm_v, &B.v_full[vs], 64 * h, rb);
          }
          ++gk;
        }
        if (aborted) break;
        cur_next_item<false>(p, c);
      }
      if (bad || c.bad) atomicOr(p.err, kErrBadIndex);
      // Drain: the last armed phase of every slot covers every copy issued.
      for (int s = 0; s < L::KS && s < gk; ++s) W.drain_wait(&B.k_full[s], (((gk - 1 - s) / L::KS)) & 1);
      for (int s = 0; s < L::VS && s < gk; ++s) W.drain_wait(&B.v_full[s], (((gk - 1 - s) / L::VS)) & 1);
      for (int s = 0; s < 2 && s < gq; ++s) W.drain_wait(&B.q_full[s], (((gq - 1 - s) / 2)) & 1);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ S (warp 1) / dP (warp 2) issuer
    regs_dec<56>();
    if (lane == 0) {
      const bool is_s = warp == 1;
      constexpr uint32_t idesc = idesc_bf16_f32(64, 128, false, false);
      const uint32_t col = is_s ? kQS : kQP;
      const int ring = is_s ? L::KS : L::VS;
      const uint64_t adesc0 = sdesc_sw128(smem_u32(tiles + (is_s ? L::OFF_Q : L::OFF_DO)), 16, 1024);
      const uint64_t bdesc0 = sdesc_sw128(smem_u32(tiles + (is_s ? L::OFF_K : L::OFF_V)), 16, 1024);
      uint64_t* full = is_s ? B.k_full : B.v_full;
      uint64_t* freed = is_s ? &B.s_free : &B.dp_free;
      uint64_t* done = is_s ? &B.s_full : &B.dp_full;
      bool aborted = false, issued = false;
      int j = 0;  // CTA step
      Cur c;
      cur_init<false>(p, c);
      while (c.live && !aborted) {
        const int qb = c.is & 1;
        const int steps = (c.n + 1) >> 1;
        for (int t = 0; t < steps; ++t) {
          const int rs = j % ring;
          // The single S (dP) buffer is free once the elementwise warps have read step j - 1.
          if ((j >= 1 && !W.wait(freed, (j - 1) & 1)) || (t == 0 && !W.wait(&B.q_full[qb], (c.is >> 1) & 1)) ||
              !W.wait(&full[rs], (j / ring) & 1)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((qb * L::TILE) >> 4);
          const uint64_t bd = bdesc0 + (uint64_t)((rs * L::PAIR) >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)  // steps of 16 along D
            mma_bf16_ss(tmem + col, ad + kmajor_off(k), bd + (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                        idesc, k > 0 ? 1u : 0u);
          mma_commit(done);
          if (!is_s) mma_commit(&B.v_empty[rs]);
          if (t == steps - 1) mma_commit(&B.q_empty[qb]);
          issued = true;
          ++j;
        }
        if (aborted) break;
        cur_next_item<false>(p, c);
      }
      if (issued) {
        mma_commit(&B.drain[warp - 1]);
        W.drain_wait(&B.drain[warp - 1], 0);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ dQ issuer
    regs_dec<56>();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(64, D, false, true);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_K), 16384, 1024);  // MN-major K pair
      bool aborted = false, issued = false;
      int j = 0;  // CTA step; dS buffer j % 2, its use j / 2
      Cur c;
      cur_init<false>(p, c);
      while (c.live && !aborted) {
        const int steps = (c.n + 1) >> 1;
        for (int t = 0; t < steps; ++t) {
          const int ks = j % L::KS, d = j & 1;
          if ((t == 0 && c.is >= 1 && !W.wait(&B.acc_empty, (c.is - 1) & 1)) ||
              !W.wait(&B.ds_full[d], (j >> 1) & 1)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)((ks * L::PAIR) >> 4);
#pragma unroll
          for (int k = 0; k < 8; ++k)  // 8 slices of 16 keys
            mma_bf16_ts(tmem + kQAcc, tmem + kQdS + 64u * d + packed_col(k), kd + (uint64_t)((k * 2048) >> 4), idesc,
                        (t > 0 || k > 0) ? 1u : 0u);
          mma_commit(&B.ds_free[d]);
          mma_commit(&B.k_empty[ks]);
          if (t == steps - 1) mma_commit(&B.acc_full);
          issued = true;
          ++j;
        }
        if (aborted) break;
        cur_next_item<false>(p, c);
      }
      if (issued) {
        mma_commit(&B.drain[2]);
        W.drain_wait(&B.drain[2], 0);
      }
    }
    __syncwarp();
  } else if (warp < 12) {
    // ------------------------------------------------------------ P, dS
    // Warp w: lane quarter w % 4 (rows), key half (w - 4) / 4 of every step.
    const int quarter = warp & 3, hf = (warp - 4) >> 2;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);
    const float sl2 = p.scale_log2;
    int j = 0;  // CTA step
    Cur c;
    cur_init<false>(p, c);
    while (c.live) {
      const int qb = c.is & 1;
      W.wait(&B.q_full[qb], (c.is >> 1) & 1);
      const float* stat = reinterpret_cast<const float*>(tiles + L::OFF_STAT + qb * 512);
      const float l0 = stat[ra], l1 = stat[ra + 8], d0 = stat[64 + ra], d1 = stat[64 + ra + 8];
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.q_empty[qb]);
      const int steps = (c.n + 1) >> 1;
      for (int t = 0; t < steps; ++t, ++j) {
        const int d = j & 1, ud = j >> 1;  // dS buffer and its use
        W.wait(&B.s_full, j & 1);
        W.wait(&B.dp_full, j & 1);
        tc_fence_after();
        uint32_t sr[32], g[32];
        tmem_ld16x256b_x8(tmem + lane_base + kQS + 64u * hf, sr);
        tmem_ld16x256b_x8(tmem + lane_base + kQP + 64u * hf, g);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.s_free);
          mbar_arrive(&B.dp_free);
        }
        uint32_t pk_p[16], pk_s[16];
        p_ds<true>(sr, g, sl2, l0, l1, d0, d1, nullptr, nullptr, 0, pk_p, pk_s);
        if (hf == 1 && 2 * t + 1 >= c.n) {
          // odd tail: keys 64..127 repeat the last cube and do not take part
#pragma unroll
          for (int e = 0; e < 16; ++e) pk_s[e] = 0u;
        }
        // dS buffer d is free once the dQ product of step j - 2 completed
        if (ud >= 1) W.wait(&B.ds_free[d], (ud - 1) & 1);
        tc_fence_after();
        tmem_st16x128b_x8(tmem + lane_base + kQdS + 64u * d + 32u * hf, pk_s);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.ds_full[d]);
      }
      cur_next_item<false>(p, c);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    regs_inc<200>();
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);
    const int tq = lane & 3;
    const int est = tid - 384;
    uint8_t* stage = tiles + L::OFF_STAGE;
    const int Hc = p.H >> 2, Wc = p.W >> 2;
    auto prefetch = [&](int is) {
      const int item = item_at(p, is);
      if (item >= 0 && est < D / 4) cp_async16(&sh.cpre[is & 1][4 * est], p.cpart0 + (size_t)item * D + 4 * est);
      cp_async_commit();
    };
    prefetch(0);
    for (int is = 0; item_at(p, is) >= 0; ++is) {
      const int item = item_at(p, is);
      const int bh = item / C, ci = item - bh * C;
      const int ct = ci / (Hc * Wc), ch = (ci / Wc) % Hc, cw = ci % Wc;
      prefetch(is + 1);
      W.wait(&B.acc_full, is & 1);
      tc_fence_after();
      float o[2 * D / 4];
      load_acc<D>(tmem + lane_base + kQAcc, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.acc_empty);
      cp_async_wait<1>();
      if (est == 0) bulk_wait_read0();
      epi_sync();
      store_tile<D>(o, p.scale, sh.cpre[is & 1], stage, ra, tq, est, &p.tm_out0, ct, ch, cw, bh);
    }
    cp_async_wait<0>();
    if (est == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================ dK/dV kernel
template <int D>
struct DkvL {
  static constexpr int NH = D / 64;
  static constexpr int TILE = 64 * D * 2;
  static constexpr int RS = 4;                              // ring of (Q, dO, statistics) steps
  static constexpr int SLOT = 2 * TILE + 1024;              // Q, dO, statistics (512 B, padded)
  static constexpr int OFF_KV = 0;                          // [2][K, V]
  static constexpr int OFF_RING = OFF_KV + 4 * TILE;
  static constexpr int OFF_STAGE = OFF_RING + RS * SLOT;
  static constexpr int BYTES = OFF_STAGE + TILE;
  static constexpr int SMEM = BYTES + 1024;
};
// dK/dV kernel tensor memory: one fp32 S^T and one fp32 dP^T buffer (64
// columns each), released as soon as the elementwise warps have read them;
// two bf16 buffers of P^T and dS^T (64 columns: P^T at +0, dS^T at +32; step
// j uses j % 2, written by group j % 2), released by the dV / dK products;
// dK and dV accumulators (D columns each).
constexpr uint32_t kTS = 0, kTP = 64, kTPD = 128, kTAcc = 256;

struct __align__(8) DkvBars {
  uint64_t kv_full[2], kv_empty[2];
  uint64_t r_full[4], r_empty[4];
  // S^T and dP^T of step g complete on st_full[g % 2] / dpt_full[g % 2]: each
  // elementwise group waits on its own barrier (a parity wait on a barrier
  // that completes for both groups in turn could not tell its phase from the
  // previous one). The buffers are freed in step order (one waiter each).
  uint64_t st_full[2], dpt_full[2], st_free, dpt_free;
  uint64_t pd_full[2], pd_free[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain[3];
};
struct alignas(16) DkvShared {
  DkvBars bar;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float cpre[2][2][128];  // [item parity][dk_bar, dv_bar] rows
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) fine_dkv_kernel(const __grid_constant__ BwdFineParams p) {
  using L = DkvL<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ DkvShared sh;
  DkvBars& B = sh.bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Waiter W{&sh.abort_flag, p.err, p.wait_ns};
  const int C = p.C;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&B.kv_full[i], 1); mbar_init(&B.kv_empty[i], 2); }
    for (int i = 0; i < L::RS; ++i) { mbar_init(&B.r_full[i], 1); mbar_init(&B.r_empty[i], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.st_full[b], 1);
      mbar_init(&B.dpt_full[b], 1);
    }
    mbar_init(&B.st_free, 4);
    mbar_init(&B.dpt_free, 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.pd_full[b], 4);
      mbar_init(&B.pd_free[b], 1);
    }
    mbar_init(&B.acc_full, 1);
    mbar_init(&B.acc_empty, 4);
    for (int i = 0; i < 3; ++i) mbar_init(&B.drain[i], 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_do);
    prefetch_tmap(&p.tm_out0);
    prefetch_tmap(&p.tm_out1);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    regs_dec<56>();
    if (lane == 0) {
      bool aborted = false, bad = false;
      int g = 0, kvu = 0;  // ring steps armed, items with steps (K/V loads)
      Cur c;
      cur_init<true>(p, c);
      while (c.live && !aborted) {
        if (c.n > 0) {
          const int kb = kvu & 1;
          if (kvu >= 2 && !W.wait(&B.kv_empty[kb], ((kvu >> 1) - 1) & 1)) { aborted = true; break; }
          mbar_arrive_expect_tx(&B.kv_full[kb], 2 * L::TILE);
          uint8_t* kvb = tiles + L::OFF_KV + kb * 2 * L::TILE;
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(kvb + h * 8192, &p.tm_k, &B.kv_full[kb], 64 * h, c.item * 64);
            tma_load_2d(kvb + L::TILE + h * 8192, &p.tm_v, &B.kv_full[kb], 64 * h, c.item * 64);
          }
          ++kvu;
          const int bh = c.item / C;
          const int32_t* lst = p.list + p.off[c.item];
          for (int t = 0; t < c.n; ++t) {
            int i = lst[t];
            if (i < 0 || i >= C) { bad = true; i = 0; }
            const int qrow = (bh * C + i) * 64;
            const int rs = g % L::RS;
            if (g >= L::RS && !W.wait(&B.r_empty[rs], ((g / L::RS) - 1) & 1)) { aborted = true; break; }
            uint8_t* slot = tiles + L::OFF_RING + rs * L::SLOT;
            mbar_arrive_expect_tx(&B.r_full[rs], 2 * L::TILE + 512);
            for (int h = 0; h < L::NH; ++h) {
              tma_load_2d(slot + h * 8192, &p.tm_q, &B.r_full[rs], 64 * h, qrow);
              tma_load_2d(slot + L::TILE + h * 8192, &p.tm_do, &B.r_full[rs], 64 * h, qrow);
            }
            bulk_load(slot + 2 * L::TILE, p.qstat + (size_t)(bh * C + i) * 128, 512, &B.r_full[rs]);
            ++g;
          }
          if (aborted) break;
        }
        cur_next_item<true>(p, c);
      }
      if (bad) atomicOr(p.err, kErrBadIndex);
      for (int s = 0; s < L::RS && s < g; ++s) W.drain_wait(&B.r_full[s], (((g - 1 - s) / L::RS)) & 1);
      for (int s = 0; s < 2 && s < kvu; ++s) W.drain_wait(&B.kv_full[s], (((kvu - 1 - s) / 2)) & 1);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ S^T (warp 1) / dP^T (warp 2) issuer
    regs_dec<56>();
    if (lane == 0) {
      const bool is_s = warp == 1;
      constexpr uint32_t idesc = idesc_bf16_f32(64, 64, false, false);
      const uint32_t col0 = is_s ? kTS : kTP;
      // A: K (or V) of the item; B: Q (or dO) of the step, both K-major.
      const uint64_t adesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_KV + (is_s ? 0 : L::TILE)), 16, 1024);
      const uint64_t bdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_RING + (is_s ? 0 : L::TILE)), 16, 1024);
      uint64_t* done = is_s ? B.st_full : B.dpt_full;
      uint64_t* freed = is_s ? &B.st_free : &B.dpt_free;
      bool aborted = false, issued = false;
      int g = 0, kvu = 0;  // CTA step, items with steps
      Cur c;
      cur_init<true>(p, c);
      while (c.live && !aborted) {
        if (c.n > 0) {
          const int kb = kvu & 1;
          for (int t = 0; t < c.n; ++t) {
            const int rs = g % L::RS;
            // the single fp32 buffer is free once step g - 1 was read
            if ((t == 0 && !W.wait(&B.kv_full[kb], (kvu >> 1) & 1)) ||
                (g >= 1 && !W.wait(freed, (g - 1) & 1)) || !W.wait(&B.r_full[rs], (g / L::RS) & 1)) {
              aborted = true;
              break;
            }
            tc_fence_after();
            const uint64_t ad = adesc0 + (uint64_t)((kb * 2 * L::TILE) >> 4);
            const uint64_t bd = bdesc0 + (uint64_t)((rs * L::SLOT) >> 4);
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              mma_bf16_ss(tmem + col0, ad + kmajor_off(k), bd + kmajor_off(k), idesc, k > 0 ? 1u : 0u);
            mma_commit(&done[g & 1]);
            if (t == c.n - 1) mma_commit(&B.kv_empty[kb]);
            issued = true;
            ++g;
          }
          if (aborted) break;
          ++kvu;
        }
        cur_next_item<true>(p, c);
      }
      if (issued) {
        mma_commit(&B.drain[warp - 1]);
        W.drain_wait(&B.drain[warp - 1], 0);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ dV / dK issuer
    regs_dec<56>();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(64, D, false, true);
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_RING), 8192, 1024);            // MN-major Q
      const uint64_t ddesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_RING + L::TILE), 8192, 1024);  // MN-major dO
      bool aborted = false, issued = false;
      int g = 0, acc = 0;  // CTA step, items with steps
      Cur c;
      cur_init<true>(p, c);
      while (c.live && !aborted) {
        if (c.n > 0) {
          for (int t = 0; t < c.n; ++t) {
            const int rs = g % L::RS, b = g & 1;
            if ((t == 0 && acc >= 1 && !W.wait(&B.acc_empty, (acc - 1) & 1)) || !W.wait(&B.pd_full[b], (g >> 1) & 1)) {
              aborted = true;
              break;
            }
            tc_fence_after();
            const uint64_t so = (uint64_t)((rs * L::SLOT) >> 4);
            const uint32_t pd = tmem + kTPD + 64u * b;
#pragma unroll
            for (int k = 0; k < 4; ++k)  // dV += P^T dO
              mma_bf16_ts(tmem + kTAcc + D, pd + packed_col(k), ddesc0 + so + (uint64_t)((k * 2048) >> 4), idesc,
                          (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // dK += dS^T Q
              mma_bf16_ts(tmem + kTAcc, pd + 32u + packed_col(k), qdesc0 + so + (uint64_t)((k * 2048) >> 4), idesc,
                          (t > 0 || k > 0) ? 1u : 0u);
            mma_commit(&B.pd_free[b]);
            mma_commit(&B.r_empty[rs]);
            if (t == c.n - 1) mma_commit(&B.acc_full);
            issued = true;
            ++g;
          }
          if (aborted) break;
          ++acc;
        }
        cur_next_item<true>(p, c);
      }
      if (issued) {
        mma_commit(&B.drain[2]);
        W.drain_wait(&B.drain[2], 0);
      }
    }
    __syncwarp();
  } else if (warp < 12) {
    // ------------------------------------------------------------ P^T, dS^T
    // Group grp takes the steps g with g % 2 == grp (bf16 buffer grp).
    const int quarter = warp & 3, grp = (warp - 4) >> 2;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int c0 = 2 * (lane & 3);  // first query column of the thread (plus 8 j)
    const float sl2 = p.scale_log2;
    int g = 0;
    Cur c;
    cur_init<true>(p, c);
    while (c.live) {
      for (int t = 0; t < c.n; ++t, ++g) {
        if ((g & 1) != grp) continue;
        const int rs = g % L::RS;
        W.wait(&B.r_full[rs], (g / L::RS) & 1);
        W.wait(&B.st_full[grp], (g >> 1) & 1);
        W.wait(&B.dpt_full[grp], (g >> 1) & 1);
        tc_fence_after();
        const float* stat = reinterpret_cast<const float*>(tiles + L::OFF_RING + rs * L::SLOT + 2 * L::TILE);
        uint32_t s[32], gg[32];
        tmem_ld16x256b_x8(tmem + lane_base + kTS, s);
        tmem_ld16x256b_x8(tmem + lane_base + kTP, gg);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.st_free);
          mbar_arrive(&B.dpt_free);
        }
        uint32_t pk_p[16], pk_s[16];
        p_ds<false>(s, gg, sl2, 0.f, 0.f, 0.f, 0.f, stat, stat + 64, c0, pk_p, pk_s);
        // bf16 buffer grp is free once the dV / dK products of step g - 2 completed
        if (g >= 2) W.wait(&B.pd_free[grp], ((g >> 1) - 1) & 1);
        tc_fence_after();
        tmem_st16x128b_x8(tmem + lane_base + kTPD + 64u * grp, pk_p);
        tmem_st16x128b_x8(tmem + lane_base + kTPD + 64u * grp + 32u, pk_s);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.pd_full[grp]);
      }
      cur_next_item<true>(p, c);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    regs_inc<200>();
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);
    const int tq = lane & 3;
    const int est = tid - 384;
    uint8_t* stage = tiles + L::OFF_STAGE;
    const int Hc = p.H >> 2, Wc = p.W >> 2;
    auto prefetch = [&](int is) {
      const int item = item_at(p, is);
      if (item >= 0 && est < D / 2) {
        const int which = est / (D / 4), e = est % (D / 4);
        cp_async16(&sh.cpre[is & 1][which][4 * e], (which ? p.cpart1 : p.cpart0) + (size_t)item * D + 4 * e);
      }
      cp_async_commit();
    };
    prefetch(0);
    int acc = 0;
    Cur c;
    cur_init<true>(p, c);
    while (c.live) {
      const int is = c.is, item = c.item;
      const int bh = item / C, kc = item - bh * C;
      const int ct = kc / (Hc * Wc), ch = (kc / Wc) % Hc, cw = kc % Wc;
      prefetch(is + 1);
      float ok[2 * D / 4], ov[2 * D / 4];
      if (c.n > 0) {
        W.wait(&B.acc_full, acc & 1);
        tc_fence_after();
        load_acc<D>(tmem + lane_base + kTAcc, ok);
        load_acc<D>(tmem + lane_base + kTAcc + D, ov);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.acc_empty);
        ++acc;
      } else {
#pragma unroll
        for (int e = 0; e < 2 * D / 4; ++e) ok[e] = ov[e] = 0.f;
      }
      cp_async_wait<1>();
      if (est == 0) bulk_wait_read0();
      epi_sync();
      store_tile<D>(ok, p.scale, sh.cpre[is & 1][0], stage, ra, tq, est, &p.tm_out0, ct, ch, cw, bh);
      if (est == 0) bulk_wait_read0();
      epi_sync();
      store_tile<D>(ov, 1.0f, sh.cpre[is & 1][1], stage, ra, tq, est, &p.tm_out1, ct, ch, cw, bh);
      cur_next_item<true>(p, c);
    }
    cp_async_wait<0>();
    if (est == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_dq_t(const BwdFineParams& p, int grid, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fine_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqL<D>::SMEM);
  if (e != cudaSuccess) return e;
  fine_dq_kernel<D><<<grid, kThreads, DqL<D>::SMEM, st>>>(p);
  return cudaGetLastError();
}
template <int D>
cudaError_t launch_dkv_t(const BwdFineParams& p, int grid, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fine_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DkvL<D>::SMEM);
  if (e != cudaSuccess) return e;
  fine_dkv_kernel<D><<<grid, kThreads, DkvL<D>::SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fine_dq(const BwdFineParams& p, int D, int grid, cudaStream_t st) {
  return D == 128 ? launch_dq_t<128>(p, grid, st) : launch_dq_t<64>(p, grid, st);
}
cudaError_t launch_fine_dkv(const BwdFineParams& p, int D, int grid, cudaStream_t st) {
  return D == 128 ? launch_dkv_t<128>(p, grid, st) : launch_dkv_t<64>(p, grid, st);
}

}  // namespace vsa
