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
// cubes of one or two heads stay resident in L2.
//
// The 64-row query tile is too short for the tensor core's 128-row M, so both
// products are computed transposed, with two selected KV cubes (128 keys)
// per step:
//   S^T[128 keys x 64 q]  = K_pair[128 x D] . Q[64 x D]^T      (tcgen05, M=128, N=64)
//   O^T[D x 64 q]        += V_pair^T[D x 128] . P^T[128 x 64]  (tcgen05, M=D,   N=64)
// Both accumulate in tensor memory (TMEM). Each softmax thread owns one key
// row of S^T (64 query columns); column statistics (the running max) are
// reduced across the 128 softmax threads only when some score exceeds the
// current reference by more than 2^8 (lazy rescaling), which after the first
// step of an item is rare. Row sums are kept as per-thread partials and
// reduced once per item.
//
// Warp roles (256 threads):
//   warp 0  TMA producer for Q and K tiles (lane 0 issues)
//   warp 1  TMA producer for V tiles (a second issuing thread doubles the
//           TMA request rate a single thread can sustain)
//   warp 2  TMEM allocation and the single-thread tcgen05.mma issuer
//   warp 3  idle
//   warps 4-7  softmax (key row = TMEM lane) and the epilogue
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

constexpr int kThreads = 256;
constexpr int kNK = 2;  // K tile stages
constexpr int kNV = 2;  // V tile stages
constexpr uint32_t kTmemCols = 256;
constexpr int kSoftmaxBar = 1;  // named barrier of the 128 softmax threads

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync %0, 128;" ::"n"(kSoftmaxBar) : "memory");
}
// Barrier over the 128 softmax threads that also ORs a predicate.
__device__ __forceinline__ bool softmax_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kSoftmaxBar)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Column-wise reduction of a 64-wide row held by each lane: after the call,
// v[0] and v[1] hold the reduction over the 32 lanes of columns 2*lane and
// 2*lane+1 (recursive halving: each stage keeps half the columns and
// exchanges the other half with the partner lane).
template <bool IS_MAX>
__device__ __forceinline__ void warp_colreduce64(float (&v)[64], int lane) {
#define VSA_STAGE(W, BIT)                                             \
  {                                                                   \
    const bool up = (lane & BIT) != 0;                                \
    _Pragma("unroll") for (int j = 0; j < W; ++j) {                   \
      const float send = up ? v[j] : v[j + W];                        \
      const float keep = up ? v[j + W] : v[j];                        \
      const float recv = __shfl_xor_sync(0xffffffffu, send, BIT);     \
      v[j] = IS_MAX ? fmaxf(keep, recv) : keep + recv;                \
    }                                                                 \
  }
  VSA_STAGE(32, 16)
  VSA_STAGE(16, 8)
  VSA_STAGE(8, 4)
  VSA_STAGE(4, 2)
  VSA_STAGE(2, 1)
#undef VSA_STAGE
}

template <int D>
struct Layout {
  static constexpr int NH = D / 64;              // 128-byte column groups of a row
  static constexpr int Q_BYTES = 64 * D * 2;     // one query cube
  static constexpr int KV_BYTES = 128 * D * 2;   // two KV cubes
  static constexpr int P_BYTES = 128 * 64 * 2;   // P^T, 128 keys x 64 queries
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + kNK * KV_BYTES;
  static constexpr int OFF_P = OFF_V + kNV * KV_BYTES;
  static constexpr int TILE_BYTES = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM_BYTES = TILE_BYTES + 1024;  // + alignment slack
};

struct __align__(8) Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full[2], o_empty[2];
  uint64_t drain, stall;
};

struct alignas(16) Shared {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float m_ref[64];   // running max per query (log2 units, scaled)
  alignas(16) float alpha[64];   // rescale factor of the last max update
  alignas(16) float red[4][64];  // per-warp column partials
  alignas(16) float inv_l[64];
  alignas(16) float gc[64];
  alignas(16) float gf[64];
  alignas(16) int tok[64];       // raster token of each query row of the item
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
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Shared sh;
  Bars& B = sh.bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Waiter W{&sh, p.err, p.wait_ns};
  const int C = p.C;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.q_full[i], 1);
      mbar_init(&B.q_empty[i], 4);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.s_empty[i], 4);
      mbar_init(&B.p_full[i], 4);
      mbar_init(&B.p_empty[i], 1);
      mbar_init(&B.o_full[i], 1);
      mbar_init(&B.o_empty[i], 4);
    }
    for (int i = 0; i < kNK; ++i) { mbar_init(&B.k_full[i], 1); mbar_init(&B.k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&B.v_full[i], 1); mbar_init(&B.v_empty[i], 1); }
    mbar_init(&B.drain, 1);
    mbar_init(&B.stall, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_q);
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
  // TMEM columns: S^T buffers at [0,64) and [64,128); O^T buffers at [128,192) and [192,256).
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------ producers
    const bool is_k = (warp == 0);
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    constexpr int NS = kNK;  // kNK == kNV
    uint8_t* ring = tiles + (is_k ? L::OFF_K : L::OFF_V);
    const CUtensorMap* tm = is_k ? &p.tm_k : &p.tm_v;
    int g = 0;                       // tiles issued
    int last_q = -1;                 // last item whose Q load was issued
    bool bad = false, aborted = false;
    for (int li = 0, item = blockIdx.x; item < p.n_items && !aborted; ++li, item += gridDim.x) {
      const int bh = item / C;
      const int n = item_count(p, item, &bad);
      const int ntiles = (n + 1) >> 1;
      const int32_t* list = p.idx + (size_t)item * p.kcap;
      if (is_k) {
        const int qb = li & 1;
        if (lane == 0) {
          if (li >= 2 && !W.wait(&B.q_empty[qb], ((li - 2) >> 1) & 1)) aborted = true;
          if (!aborted) {
            mbar_arrive_expect_tx(&B.q_full[qb], L::Q_BYTES);
            uint8_t* dst = tiles + L::OFF_Q + qb * L::Q_BYTES;
#pragma unroll
            for (int h = 0; h < L::NH; ++h) tma_load_2d(dst + h * 8192, &p.tm_q, &B.q_full[qb], 64 * h, item * 64);
            last_q = li;
          }
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
      }
      for (int t0 = 0; t0 < ntiles && !aborted; t0 += 16) {
        const int e = 2 * t0 + lane;
        int mine = (e < n) ? list[e] : 0;
        if (mine < 0 || mine >= C) {
          if (e < n) bad = true;
          mine = 0;
        }
        const int tend = min(ntiles, t0 + 16);
        for (int t = t0; t < tend; ++t, ++g) {
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
        }
      }
    }
    if (bad && lane == 0) atomicOr(p.err, kErrBadIndex);
    // Drain: wait for the copies this thread issued. Tiles 0..g-1 were
    // issued (an aborted step breaks before issuing and before ++g); only the
    // last use of each stage can still be in flight.
    if (lane == 0) {
      for (int j = max(0, g - NS); j < g; ++j) W.drain_wait(&full[j % NS], (j / NS) & 1);
      if (is_k && last_q >= 0)
        for (int lj = max(0, last_q - 1); lj <= last_q; ++lj) W.drain_wait(&B.q_full[lj & 1], (lj >> 1) & 1);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(D, 64, true, true);
      const uint32_t sQ = smem_u32(tiles + L::OFF_Q), sK = smem_u32(tiles + L::OFF_K),
                     sV = smem_u32(tiles + L::OFF_V), sP = smem_u32(tiles + L::OFF_P);
      bool aborted = false, issued_any = false, bad = false;
      if (p.debug_stall && !W.wait(&B.stall, 0)) aborted = true;
      int g = 0;
      // O^T step for tile gg (first = first tile of its item).
      auto issue_o = [&](int gg, bool first, int ob) -> bool {
        const int vs = gg % kNV, pb = gg & 1;
        if (!W.wait(&B.v_full[vs], (gg / kNV) & 1)) return false;
        if (!W.wait(&B.p_full[pb], (gg >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s) {  // 8 steps of 16 keys
          const uint64_t ad = sdesc_sw128(sV + vs * L::KV_BYTES + s * 2048, 16384, 1024);
          const uint64_t bd = sdesc_sw128(sP + pb * L::P_BYTES + s * 2048, 8192, 1024);
          mma_bf16_ss(tO + ob * 64, ad, bd, idesc_o, (first && s == 0) ? 0u : 1u);
        }
        mma_commit(&B.v_empty[vs]);
        mma_commit(&B.p_empty[pb]);
        return true;
      };
      for (int li = 0, item = blockIdx.x; item < p.n_items && !aborted; ++li, item += gridDim.x) {
        const int n = item_count(p, item, &bad);
        const int ntiles = (n + 1) >> 1;
        const int qb = li & 1, ob = li & 1;
        if (!W.wait(&B.q_full[qb], (li >> 1) & 1)) { aborted = true; break; }
        if (li >= 2 && !W.wait(&B.o_empty[ob], ((li - 2) >> 1) & 1)) { aborted = true; break; }
        for (int t = 0; t < ntiles; ++t, ++g) {
          const int ks = g % kNK, sb = g & 1;
          if (!W.wait(&B.k_full[ks], (g / kNK) & 1)) { aborted = true; break; }
          if (g >= 2 && !W.wait(&B.s_empty[sb], ((g - 2) >> 1) & 1)) { aborted = true; break; }
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < D / 16; ++s) {  // steps of 16 along D
            const uint32_t koff = (s >> 2) * 16384 + (s & 3) * 32;
            const uint32_t qoff = (s >> 2) * 8192 + (s & 3) * 32;
            const uint64_t ad = sdesc_sw128(sK + ks * L::KV_BYTES + koff, 16, 1024);
            const uint64_t bd = sdesc_sw128(sQ + qb * L::Q_BYTES + qoff, 16, 1024);
            mma_bf16_ss(tS + sb * 64, ad, bd, idesc_s, s > 0 ? 1u : 0u);
          }
          issued_any = true;
          mma_commit(&B.k_empty[ks]);
          mma_commit(&B.s_full[sb]);
          if (t > 0 && !issue_o(g - 1, t == 1, ob)) { aborted = true; break; }
        }
        if (aborted) break;
        if (!issue_o(g - 1, ntiles == 1, ob)) { aborted = true; break; }
        mma_commit(&B.o_full[ob]);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is released.
      if (issued_any) {
        mma_commit(&B.drain);
        W.drain_wait(&B.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int sw = warp - 4;              // TMEM lane quarter
    const int kr = sw * 32 + lane;        // key row of S^T / d row of O^T
    const uint32_t lane_base = (uint32_t)(sw * 32) << 16;
    const float scale = p.scale_log2;
    uint8_t* sP = tiles + L::OFF_P;
    int g = 0;
    bool bad = false;
    for (int li = 0, item = blockIdx.x; item < p.n_items; ++li, item += gridDim.x) {
      const int bh = item / C, ci = item - bh * C;
      const int n = item_count(p, item, &bad);
      const int ntiles = (n + 1) >> 1;
      const int ob = li & 1, qb = li & 1;
      const int st = kr;  // softmax-group thread index 0..127
      if (st < 64) {
        sh.m_ref[st] = -INFINITY;
        const int tok = cube_token(ci, st, p.H, p.W);
        sh.tok[st] = tok;
        sh.gc[st] = p.gate_c[(size_t)bh * p.N + tok];
        sh.gf[st] = p.gate_f[(size_t)bh * p.N + tok];
      }
      float lp[64];
#pragma unroll
      for (int q = 0; q < 64; ++q) lp[q] = 0.f;
      softmax_sync();

      for (int t = 0; t < ntiles; ++t, ++g) {
        const int sb = g & 1, pb = g & 1;
        W.wait(&B.s_full[sb], (g >> 1) & 1);
        tc_fence_after();
        float x[64];
        {
          uint32_t r[32];
          tmem_ld32(tS + sb * 64 + lane_base, r);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = __uint_as_float(r[q]) * scale;
          tmem_ld32(tS + sb * 64 + 32 + lane_base, r);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) x[32 + q] = __uint_as_float(r[q]) * scale;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.s_empty[sb]);
        const bool valid = (kr < 64) || (2 * t + 1 < n);
        // Does any score exceed the current reference max by more than 2^8?
        bool need = false;
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&sh.m_ref[4 * q4]);
          need |= (x[4 * q4 + 0] - m4.x > 8.0f) | (x[4 * q4 + 1] - m4.y > 8.0f) |
                  (x[4 * q4 + 2] - m4.z > 8.0f) | (x[4 * q4 + 3] - m4.w > 8.0f);
        }
        need = softmax_sync_or(valid && need);
        if (need) {
          // Exact column max over the 128 keys of this step -> new reference.
          float cm[64];
#pragma unroll
          for (int q = 0; q < 64; ++q) cm[q] = valid ? x[q] : -INFINITY;
          warp_colreduce64<true>(cm, lane);
          sh.red[sw][2 * lane] = cm[0];
          sh.red[sw][2 * lane + 1] = cm[1];
          softmax_sync();
          if (st < 64) {
            const float c = fmaxf(fmaxf(sh.red[0][st], sh.red[1][st]), fmaxf(sh.red[2][st], sh.red[3][st]));
            const float mo = sh.m_ref[st];
            const float mn = fmaxf(mo, c);
            sh.alpha[st] = fast_exp2(mo - mn);  // 0 when mo = -inf
            sh.m_ref[st] = mn;
          }
          softmax_sync();
#pragma unroll
          for (int q = 0; q < 64; ++q) lp[q] *= sh.alpha[q];
          if (t > 0) {
            // O^T holds steps < t of this item: rescale its query columns once
            // the previous step's MMA has completed. All lanes take part in
            // the (warp-collective) TMEM load/store.
            W.wait(&B.p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1);
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t r[32];
              const uint32_t a = tO + ob * 64 + half * 32 + lane_base;
              tmem_ld32(a, r);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * sh.alpha[half * 32 + q]);
              tmem_st32(a, r);
            }
            tmem_wait_st();
          }
        }
        // p = 2^(x - m_ref), accumulated into the row-sum partials; x is reused for p.
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&sh.m_ref[4 * q4]);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 4 * q4 + e;
            const float pq = valid ? fast_exp2(x[q] - mm[e]) : 0.f;
            lp[q] += pq;
            x[q] = pq;
          }
        }
        // P^T row kr -> shared memory (MN-major, 128-byte swizzle), once the
        // MMA that read this buffer two steps ago has completed.
        if (g >= 2) W.wait(&B.p_empty[pb], ((g - 2) >> 1) & 1);
        uint8_t* prow = sP + pb * L::P_BYTES + kr * 128;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * c8 + 2 * e], x[8 * c8 + 2 * e + 1]);
            w4[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(prow + ((c8 ^ (kr & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[pb]);
      }

      // ---------------------------------------------------------- epilogue
      warp_colreduce64<false>(lp, lane);
      sh.red[sw][2 * lane] = lp[0];
      sh.red[sw][2 * lane + 1] = lp[1];
      softmax_sync();
      if (st < 64) sh.inv_l[st] = 1.0f / (sh.red[0][st] + sh.red[1][st] + sh.red[2][st] + sh.red[3][st]);
      softmax_sync();
      W.wait(&B.o_full[ob], (li >> 1) & 1);
      tc_fence_after();
      const bool has_d = (D == 128) || (lane < 16);
      const int d = (D == 128) ? kr : sw * 16 + lane;
      float o[64];
      {
        uint32_t r[32];
        tmem_ld32(tO + ob * 64 + lane_base, r);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = __uint_as_float(r[q]);
        tmem_ld32(tO + ob * 64 + 32 + lane_base, r);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) o[32 + q] = __uint_as_float(r[q]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.o_empty[ob]);
      const float ocd = has_d ? p.oc[((size_t)bh * C + ci) * D + d] : 0.f;
#pragma unroll
      for (int q = 0; q < 64; ++q) o[q] *= sh.inv_l[q];
      if (p.out_fine && has_d) {
        for (int q = 0; q < 64; ++q) p.out_fine[((size_t)bh * p.N + sh.tok[q]) * D + d] = o[q];
      }
      uint8_t* stage = tiles + L::OFF_Q + qb * L::Q_BYTES;  // Q buffer of this item, free now
      if (p.out) {
        // Gated combine, then pair lanes (d, d+1) so each lane writes 4 bytes.
        const bool odd = lane & 1;
#pragma unroll
        for (int q2 = 0; q2 < 32; ++q2) {
          const int qa = 2 * q2, qb2 = 2 * q2 + 1;
          const float va = sh.gc[qa] * ocd + sh.gf[qa] * o[qa];
          const float vb = sh.gc[qb2] * ocd + sh.gf[qb2] * o[qb2];
          const float send = odd ? va : vb;
          const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
          if (has_d) {
            // even lane: (q=qa: d, d+1); odd lane: (q=qb2: d-1, d)
            const int q = odd ? qb2 : qa;
            const int d0 = odd ? d - 1 : d;
            const __nv_bfloat162 h = odd ? __floats2bfloat162_rn(recv, vb) : __floats2bfloat162_rn(va, recv);
            *reinterpret_cast<__nv_bfloat162*>(stage + (q * D + d0) * 2) = h;
          }
        }
      }
      softmax_sync();
      if (p.out) {
        constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
        for (int u = 0; u < (64 * CPR) / 128; ++u) {
          const int c = st + 128 * u;
          const int q = c / CPR, off = c % CPR;
          const uint4 v = *reinterpret_cast<const uint4*>(stage + (q * D + off * 8) * 2);
          *reinterpret_cast<uint4*>(p.out + ((size_t)bh * p.N + sh.tok[q]) * D + off * 8) = v;
        }
      }
      fence_proxy_async_smem();
      softmax_sync();
      if (lane == 0) mbar_arrive(&B.q_empty[qb]);
    }
    (void)bad;
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
