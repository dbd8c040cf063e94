// Block-sparse fine attention with the gated coarse/fine combine.
//
// "Faster Video Diffusion with Trainable Sparse Attention", "Approach":
// block-sparse token-level fine attention only over the selected cubes, with
// the coarse and fine outputs combined through gates, each cube mapping to
// one GPU tile. "VSA: Faster Video Diffusion with Trainable Sparse
// Attention", "Abstract (arXiv)": token-level attention only inside the
// selected tiles, in a block computing layout.
//
// One work item = one query cube (64 tokens) of one (batch, head). A
// persistent CTA per SM walks items in (batch*head)-major order so the K/V
// cubes of one or two heads stay resident in L2. Each step covers two of the
// item's selected KV cubes (128 keys):
//   S[64 q x 128 keys] = Q . K_pair^T     tcgen05.mma M=64, N=128, A = Q in TMEM
//   O[64 q x D]       += P . V_pair       tcgen05.mma M=64, N=D,   A = P in TMEM
// Shared memory bandwidth, not the tensor core, bounds this kernel (every
// selected KV cube is used by one query cube, so each K/V byte is written to
// and read from shared memory once). Keeping Q and P in tensor memory leaves
// only the K and V tiles in shared memory: 64 KB written + 64 KB read per step.
//
// The M=64 accumulators occupy 16 lanes of each 32-lane TMEM quarter; the
// 16-lane tcgen05.ld/st shapes spread those lanes over all 32 threads of a
// warp: with .16x256b a thread holds rows r and r+8 of its quarter and
// columns {8j + 2(t%4), 8j + 2(t%4) + 1}, so four threads share a row and a
// row max / row sum needs two shuffles. P is packed to bf16 pairs and written
// back with .16x128b, whose column 4j + (t%4) is exactly the pair the thread
// holds. Softmax is online per row with lazy rescaling: the reference max of a
// row moves only when a score exceeds it by more than 2^8, which after the
// first step of an item is rare; O is then rescaled in place.
//
// Warp roles (384 threads):
//   warp 0      TMA producer of K tiles (3-stage ring)
//   warp 1      TMA producer of V tiles (3-stage ring; a second issuing thread,
//               since one thread cannot keep the L2 -> SM stream full)
//   warp 2      TMEM allocation, single-thread tcgen05.mma issuer
//   warp 3      idle
//   warps 4-7   softmax (warp w reads TMEM quarter w%4)
//   warps 8-11  epilogue: loads each item's Q into TMEM, reads O, applies
//               1/l and the gates, writes the output rows
// MMA order: S(g), O(g-1), S(g+1), O(g), ... over the CTA's steps. A tcgen05
// commit covers every earlier MMA of the issuing thread, so "S(g) complete"
// implies "O(g-2) complete", which is what makes the S/P double buffer safe.
//
// Every mbarrier wait is bounded (plan wait limit). A wait that gives up
// records kErrTimeout, sets a CTA-wide abort flag that makes every later wait
// return at once, and the CTA then drains its own in-flight TMA copies and
// MMAs before releasing TMEM and exiting.
#include "sm100_ptx.cuh"
#include "vsa_common.cuh"

namespace vsa {

namespace {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S/P buffers at 0 and 128, O at 256, Q buffers at 384 and 448.
constexpr uint32_t kColS = 0, kColO = 256, kColQ = 384;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// ---- 16-lane TMEM shapes (lanes base..base+15 of the warp's quarter) ----
#define VSA_O4(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3])
#define VSA_I4(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])
// .16x256b.x16: 128 columns; r[4j..4j+3] = (row a: col c, c+1; row a+8: col c, c+1), c = 8j + 2(t%4).
__device__ __forceinline__ void ld_16x256b_x16(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : VSA_O4(0), VSA_O4(4), VSA_O4(8), VSA_O4(12), VSA_O4(16), VSA_O4(20), VSA_O4(24), VSA_O4(28),
        VSA_O4(32), VSA_O4(36), VSA_O4(40), VSA_O4(44), VSA_O4(48), VSA_O4(52), VSA_O4(56), VSA_O4(60)
      : "r"(taddr));
}
__device__ __forceinline__ void ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : VSA_O4(0), VSA_O4(4), VSA_O4(8), VSA_O4(12), VSA_O4(16), VSA_O4(20), VSA_O4(24), VSA_O4(28)
      : "r"(taddr));
}
__device__ __forceinline__ void st_16x256b_x16(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
      "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12), VSA_I4(16), VSA_I4(20), VSA_I4(24), VSA_I4(28), VSA_I4(32),
      VSA_I4(36), VSA_I4(40), VSA_I4(44), VSA_I4(48), VSA_I4(52), VSA_I4(56), VSA_I4(60)
      : "memory");
}
__device__ __forceinline__ void st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12), VSA_I4(16), VSA_I4(20), VSA_I4(24), VSA_I4(28)
      : "memory");
}
__device__ __forceinline__ void st_16x256b_x4(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12)
      : "memory");
}
// .16x128b.x16: 64 columns; r[2j] -> (row a, col 4j + t%4), r[2j+1] -> (row a+8, same col).
__device__ __forceinline__ void st_16x128b_x16(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12), VSA_I4(16), VSA_I4(20), VSA_I4(24), VSA_I4(28)
      : "memory");
}
#undef VSA_O4
#undef VSA_I4

// D[tmem] (+)= A[tmem] * B[smem]^T ; issued by a single thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D>
struct Layout {
  static constexpr int NH = D / 64;              // 128-byte column groups of a row
  static constexpr int KV_BYTES = 128 * D * 2;   // two KV cubes
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + kKStages * KV_BYTES;
  static constexpr int OFF_STAGE = OFF_V + kVStages * KV_BYTES;   // output staging, 64 x D bf16
  static constexpr int TILE_BYTES = OFF_STAGE + 64 * D * 2;
  static constexpr int SMEM_BYTES = TILE_BYTES + 1024;            // + alignment slack
};

struct __align__(8) Bars {
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t q_full[2];      // epilogue warps -> MMA: Q of the item in TMEM (count 4)
  uint64_t s_full[2];      // MMA -> softmax: S of a step (commit)
  uint64_t p_full[2];      // softmax -> MMA: P of a step in TMEM (count 4)
  uint64_t l_full[2];      // softmax -> epilogue: 1/l of an item (count 4)
  uint64_t o_step;         // MMA: each O step completed (commit)
  uint64_t o_full;         // MMA -> epilogue: last O step of an item (commit)
  uint64_t o_empty;        // epilogue -> MMA: O read out (count 4)
  uint64_t drain, stall;
};

struct alignas(16) Shared {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float inv_l[2][64];
};

struct Waiter {
  Shared* sh;
  int* err;
  uint64_t limit;
  // Bounded wait; returns false (and raises the CTA abort flag) on timeout or
  // if another thread already aborted.
  __device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 64; ++i)
        if (mbar_try_wait(bar, parity)) return true;
      if (*(volatile int*)&sh->abort_flag) return false;
      if (globaltimer_ns() - t0 > limit) {
        *(volatile int*)&sh->abort_flag = 1;
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
  // Bounded wait that ignores the abort flag (used while draining).
  __device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) const {
    mbar_wait(bar, parity, limit);
  }
};

__device__ __forceinline__ int item_count(const FineParams& p, int item, bool* bad) {
  int n = p.cnt ? p.cnt[item] : p.kcap;
  if (n < 1 || n > p.kcap) {
    *bad = true;
    n = n < 1 ? 1 : p.kcap;
  }
  return n;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) fine_attention_kernel(const __grid_constant__ FineParams p) {
  using L = Layout<D>;
  constexpr uint32_t kQCols = D / 2;  // Q in TMEM: bf16 pairs
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Shared sh;
  Bars& B = sh.bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Waiter W{&sh, p.err, p.wait_ns};
  const int C = p.C;

  if (tid == 0) {
    for (int i = 0; i < kKStages; ++i) { mbar_init(&B.k_full[i], 1); mbar_init(&B.k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&B.v_full[i], 1); mbar_init(&B.v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.q_full[i], 4);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.p_full[i], 4);
      mbar_init(&B.l_full[i], 4);
    }
    mbar_init(&B.o_step, 1);
    mbar_init(&B.o_full, 1);
    mbar_init(&B.o_empty, 4);
    mbar_init(&B.drain, 1);
    mbar_init(&B.stall, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  if (warp == 2) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------ K / V producers
    const bool is_k = (warp == 0);
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    constexpr int NS = kKStages;  // == kVStages
    uint8_t* ring = tiles + (is_k ? L::OFF_K : L::OFF_V);
    const CUtensorMap* tm = is_k ? &p.tm_k : &p.tm_v;
    bool bad = false, aborted = false;
    int g = 0;  // steps issued
    for (int item = blockIdx.x; item < p.n_items && !aborted; item += gridDim.x) {
      const int bh = item / C;
      const int n = item_count(p, item, &bad);
      const int ntiles = (n + 1) >> 1;
      const int32_t* list = p.idx + (size_t)item * p.kcap;
      for (int t0 = 0; t0 < ntiles && !aborted; t0 += 16) {
        const int e = 2 * t0 + lane;
        int mine = (e < n) ? list[e] : 0;
        if (mine < 0 || mine >= C) {
          if (e < n) bad = true;
          mine = 0;
        }
        const int tend = min(ntiles, t0 + 16);
        for (int t = t0; t < tend; ++t) {
          const int ca = __shfl_sync(0xffffffffu, mine, 2 * (t - t0));
          int cb = __shfl_sync(0xffffffffu, mine, 2 * (t - t0) + 1);
          if (2 * t + 1 >= n) cb = ca;  // odd tail: load a copy, the softmax masks it
          if (lane == 0) {
            const int s = g % NS;
            if (g >= NS && !W.wait(&empty[s], ((g / NS) - 1) & 1)) aborted = true;
            if (!aborted) {
              mbar_arrive_expect_tx(&full[s], L::KV_BYTES);
              uint8_t* dst = ring + s * L::KV_BYTES;
#pragma unroll
              for (int h = 0; h < L::NH; ++h) {
                tma_load_2d(dst + h * 16384, tm, &full[s], 64 * h, (bh * C + ca) * 64);
                tma_load_2d(dst + h * 16384 + 8192, tm, &full[s], 64 * h, (bh * C + cb) * 64);
              }
            }
          }
          aborted = __shfl_sync(0xffffffffu, aborted, 0);
          if (aborted) break;
          ++g;
        }
      }
    }
    if (bad && lane == 0) atomicOr(p.err, kErrBadIndex);
    // Drain: steps 0..g-1 were issued; only the last use of each stage can be in flight.
    if (lane == 0)
      for (int j = max(0, g - NS); j < g; ++j) W.drain_wait(&full[j % NS], (j / NS) & 1);
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(64, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(64, D, false, true);
      const uint32_t sK = smem_u32(tiles + L::OFF_K), sV = smem_u32(tiles + L::OFF_V);
      // K tile: K-major (rows = keys, 128 B per row segment); V tile: MN-major (rows = keys).
      const uint64_t kdesc0 = sdesc_sw128(sK, 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(sV, 16384, 1024);
      bool aborted = false, issued_any = false, bad = false;
      if (p.debug_stall && !W.wait(&B.stall, 0)) aborted = true;
      int g = 0;          // steps (S) issued
      int li = 0;         // local item index
      // The pending O step (issued after the next S).
      bool have_prev = false, prev_first = false, prev_last = false;
      int prev_g = 0, prev_li = 0;
      auto issue_o = [&](int gg, bool first, bool last, int item_li) -> bool {
        const int vs = gg % kVStages, pb = gg & 1;
        if (!W.wait(&B.v_full[vs], (gg / kVStages) & 1)) return false;
        if (!W.wait(&B.p_full[pb], (gg >> 1) & 1)) return false;
        if (first && item_li >= 1 && !W.wait(&B.o_empty, (item_li - 1) & 1)) return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + (uint64_t)((vs * L::KV_BYTES) >> 4);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // 8 steps of 16 keys; P step s = 8 TMEM columns
          mma_bf16_ts(tmem + kColO, tmem + kColS + 128u * pb + 8u * s, vd + (uint64_t)((s * 2048) >> 4), idesc_o,
                      (first && s == 0) ? 0u : 1u);
        mma_commit(&B.v_empty[vs]);
        mma_commit(&B.o_step);
        if (last) mma_commit(&B.o_full);
        return true;
      };
      for (int item = blockIdx.x; item < p.n_items && !aborted; item += gridDim.x, ++li) {
        const int n = item_count(p, item, &bad);
        const int ntiles = (n + 1) >> 1;
        const int qb = li & 1;
        for (int t = 0; t < ntiles; ++t, ++g) {
          if (t == 0 && !W.wait(&B.q_full[qb], (li >> 1) & 1)) { aborted = true; break; }
          const int ks = g % kKStages, sb = g & 1;
          if (!W.wait(&B.k_full[ks], (g / kKStages) & 1)) { aborted = true; break; }
          tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)((ks * L::KV_BYTES) >> 4);
#pragma unroll
          for (int s = 0; s < D / 16; ++s)  // steps of 16 along D; Q step s = 8 TMEM columns
            mma_bf16_ts(tmem + kColS + 128u * sb, tmem + kColQ + kQCols * qb + 8u * s,
                        kd + (uint64_t)(((s >> 2) * 16384 + (s & 3) * 32) >> 4), idesc_s, s > 0 ? 1u : 0u);
          issued_any = true;
          mma_commit(&B.k_empty[ks]);
          mma_commit(&B.s_full[sb]);
          if (have_prev && !issue_o(prev_g, prev_first, prev_last, prev_li)) { aborted = true; break; }
          have_prev = true;
          prev_g = g;
          prev_first = (t == 0);
          prev_last = (t == ntiles - 1);
          prev_li = li;
        }
      }
      if (!aborted && have_prev && !issue_o(prev_g, prev_first, prev_last, prev_li)) aborted = true;
      // Drain: every MMA issued by this thread completes before TMEM is released.
      if (issued_any) {
        mma_commit(&B.drain);
        W.drain_wait(&B.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float scale = p.scale_log2;
    bool bad = false;
    int g = 0;
    int li = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++li) {
      const int n = item_count(p, item, &bad);
      const int ntiles = (n + 1) >> 1;
      float m0 = -INFINITY, m1 = -INFINITY;  // reference max (scaled) of rows a and a+8
      float l0 = 0.f, l1 = 0.f;              // this thread's share of the row sums
      for (int t = 0; t < ntiles; ++t, ++g) {
        const int sb = g & 1;
        W.wait(&B.s_full[sb], (g >> 1) & 1);
        tc_fence_after();
        uint32_t r[64];
        ld_16x256b_x16(tmem + kColS + 128u * sb + lane_base, r);
        tmem_wait_ld();
        const bool hi_valid = (2 * t + 1 < n);  // keys 64..127 (second cube) present
        float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < 8 || hi_valid) {
            x0 = fmaxf(x0, fmaxf(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])));
            x1 = fmaxf(x1, fmaxf(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
          }
        }
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2)) * scale;
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2)) * scale;
        // Lazy reference update per row.
        float a0 = 1.f, a1 = 1.f;
        const bool u0 = x0 > m0 + 8.0f, u1 = x1 > m1 + 8.0f;
        if (u0) { a0 = fast_exp2(m0 - x0); m0 = x0; l0 *= a0; }
        if (u1) { a1 = fast_exp2(m1 - x1); m1 = x1; l1 *= a1; }
        if (t > 0 && __any_sync(0xffffffffu, u0 || u1)) {
          // O holds steps < t of this item: wait for the previous O step, rescale rows.
          W.wait(&B.o_step, (g - 1) & 1);
          tc_fence_after();
          uint32_t o[64];
          if (D == 128) ld_16x256b_x16(tmem + kColO + lane_base, o);
          else ld_16x256b_x8(tmem + kColO + lane_base, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < D / 8; ++j) {
            o[4 * j] = __float_as_uint(__uint_as_float(o[4 * j]) * a0);
            o[4 * j + 1] = __float_as_uint(__uint_as_float(o[4 * j + 1]) * a0);
            o[4 * j + 2] = __float_as_uint(__uint_as_float(o[4 * j + 2]) * a1);
            o[4 * j + 3] = __float_as_uint(__uint_as_float(o[4 * j + 3]) * a1);
          }
          if (D == 128) st_16x256b_x16(tmem + kColO + lane_base, o);
          else st_16x256b_x8(tmem + kColO + lane_base, o);
          tmem_wait_st();
        }
        // P = 2^(s*scale - m), packed to bf16 pairs (keys c, c+1 -> P column c/2).
        uint32_t pk[32];
        const float nm0 = -m0, nm1 = -m1;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool v = (j < 8) || hi_valid;
          const float p00 = v ? fast_exp2(fmaf(__uint_as_float(r[4 * j]), scale, nm0)) : 0.f;
          const float p01 = v ? fast_exp2(fmaf(__uint_as_float(r[4 * j + 1]), scale, nm0)) : 0.f;
          const float p10 = v ? fast_exp2(fmaf(__uint_as_float(r[4 * j + 2]), scale, nm1)) : 0.f;
          const float p11 = v ? fast_exp2(fmaf(__uint_as_float(r[4 * j + 3]), scale, nm1)) : 0.f;
          l0 += p00 + p01;
          l1 += p10 + p11;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(p00, p01);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(p10, p11);
          pk[2 * j] = *reinterpret_cast<uint32_t*>(&h0);
          pk[2 * j + 1] = *reinterpret_cast<uint32_t*>(&h1);
        }
        st_16x128b_x16(tmem + kColS + 128u * sb + lane_base, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[sb]);
      }
      // Row sums of the item -> 1/l for the epilogue.
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if ((lane & 3) == 0) {
        const int row = quarter * 16 + (lane >> 2);
        sh.inv_l[li & 1][row] = 1.0f / l0;
        sh.inv_l[li & 1][row + 8] = 1.0f / l1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.l_full[li & 1]);
    }
    if (bad && tid == 128) atomicOr(p.err, kErrBadIndex);
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue (+ Q loads)
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);  // rows ra and ra + 8 of the item
    const int tq = lane & 3;
    const int est = tid - 256;                  // 0..127 within the epilogue group
    uint8_t* stage = tiles + L::OFF_STAGE;
    // Q of an item -> TMEM buffer b (A operand layout: row per lane, bf16 pairs per column).
    auto load_q = [&](int item, int b) {
      const __nv_bfloat16* qsrc = p.q_cube + (size_t)item * 64 * D;
      uint32_t r[64];
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const uint2 va = *reinterpret_cast<const uint2*>(qsrc + (size_t)ra * D + 16 * j + 4 * tq);
        const uint2 vb = *reinterpret_cast<const uint2*>(qsrc + (size_t)(ra + 8) * D + 16 * j + 4 * tq);
        r[4 * j] = va.x; r[4 * j + 1] = va.y; r[4 * j + 2] = vb.x; r[4 * j + 3] = vb.y;
      }
      const uint32_t ta = tmem + kColQ + (uint32_t)(D / 2) * b + lane_base;
      if (D == 128) st_16x256b_x8(ta, r);
      else st_16x256b_x4(ta, reinterpret_cast<uint32_t(&)[32]>(r));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.q_full[b]);
    };
    if (blockIdx.x < p.n_items) load_q(blockIdx.x, 0);
    if (blockIdx.x + gridDim.x < p.n_items) load_q(blockIdx.x + gridDim.x, 1);
    int li = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++li) {
      const int bh = item / C, ci = item - bh * C;
      // per-item constants: gates of rows ra, ra+8 and this thread's coarse-output columns
      const int tok0 = cube_token(ci, ra, p.H, p.W), tok1 = cube_token(ci, ra + 8, p.H, p.W);
      const float gc0 = p.gate_c[(size_t)bh * p.N + tok0], gf0 = p.gate_f[(size_t)bh * p.N + tok0];
      const float gc1 = p.gate_c[(size_t)bh * p.N + tok1], gf1 = p.gate_f[(size_t)bh * p.N + tok1];
      const float* ocrow = p.oc + ((size_t)bh * C + ci) * D;
      W.wait(&B.l_full[li & 1], (li >> 1) & 1);
      const float il0 = sh.inv_l[li & 1][ra], il1 = sh.inv_l[li & 1][ra + 8];
      W.wait(&B.o_full, li & 1);
      tc_fence_after();
      uint32_t o[64];
      if (D == 128) ld_16x256b_x16(tmem + kColO + lane_base, o);
      else ld_16x256b_x8(tmem + kColO + lane_base, o);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.o_empty);
      // All S steps of this item are complete, so its Q buffer takes the item after next.
      if (item + 2 * gridDim.x < p.n_items) load_q(item + 2 * gridDim.x, li & 1);
      if (p.out_fine) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const int d = 8 * j + 2 * tq;
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok0) * D + d) =
              make_float2(__uint_as_float(o[4 * j]) * il0, __uint_as_float(o[4 * j + 1]) * il0);
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok1) * D + d) =
              make_float2(__uint_as_float(o[4 * j + 2]) * il1, __uint_as_float(o[4 * j + 3]) * il1);
        }
      }
      if (p.out) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const int d = 8 * j + 2 * tq;
          const float2 oc = *reinterpret_cast<const float2*>(ocrow + d);
          const __nv_bfloat162 h0 = __floats2bfloat162_rn(gc0 * oc.x + gf0 * __uint_as_float(o[4 * j]) * il0,
                                                          gc0 * oc.y + gf0 * __uint_as_float(o[4 * j + 1]) * il0);
          const __nv_bfloat162 h1 = __floats2bfloat162_rn(gc1 * oc.x + gf1 * __uint_as_float(o[4 * j + 2]) * il1,
                                                          gc1 * oc.y + gf1 * __uint_as_float(o[4 * j + 3]) * il1);
          *reinterpret_cast<__nv_bfloat162*>(stage + (ra * D + d) * 2) = h0;
          *reinterpret_cast<__nv_bfloat162*>(stage + ((ra + 8) * D + d) * 2) = h1;
        }
        epi_sync();
        constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
        for (int u = 0; u < (64 * CPR) / 128; ++u) {
          const int cidx = est + 128 * u;
          const int q = cidx / CPR, off = cidx % CPR;
          const uint4 v = *reinterpret_cast<const uint4*>(stage + (q * D + off * 8) * 2);
          *reinterpret_cast<uint4*>(p.out + ((size_t)bh * p.N + cube_token(ci, q, p.H, p.W)) * D + off * 8) = v;
        }
        epi_sync();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_fine_t(const FineParams& p, int grid, cudaStream_t st) {
  using L = Layout<D>;
  cudaError_t e = cudaFuncSetAttribute(fine_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  fine_attention_kernel<D><<<grid, kThreads, L::SMEM_BYTES, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fine(const FineParams& p, int D, int grid, cudaStream_t st) {
  return D == 128 ? launch_fine_t<128>(p, grid, st) : launch_fine_t<64>(p, grid, st);
}

}  // namespace vsa
