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
// cubes of one or two heads stay resident in L2. Each step covers two of an
// item's selected KV cubes (128 keys):
//   S[64 q x 128 keys] = Q . K_pair^T     tcgen05.mma M=64, N=128 (Q, K in smem)
//   O[64 q x D]       += P . V_pair       tcgen05.mma M=64, N=D   (P in TMEM, V in smem)
// Each query cube is read once, straight from the raster q, by the epilogue
// warps with 16-byte cp.async copies into the 128-byte-swizzled tile (64 rows
// in in-cube slot order): the load/store path, not the TMA unit, which then
// serves only the K/V tiles (a raster box from HBM on the TMA unit held up the
// K/V tiles queued behind it). K and V cubes, read about K times each from L2,
// come from the cube-major copies (one contiguous 64 x D tile per cube) as
// 2-D TMA boxes, which load faster than strided raster boxes.
//
// Tensor memory holds three S/P buffers and the O accumulator: S of steps
// j+1 and j+2 can run on the tensor core while the softmax works on step j,
// so the chain softmax -> O MMA -> S MMA (which must wait for the O MMA that
// read the buffer's P) spans three steps. The epilogue reads an item's O as
// soon as its last MMA completes; the next item's first O MMA waits for that
// read only. All eight softmax warps work on the same step: warp w handles the
// rows of TMEM lane quarter w % 4 and the key half w / 4 (64 keys). The two
// warps that share rows agree on the row statistics through a 64-thread
// named barrier.
//
// The M=64 accumulators occupy 16 lanes of each 32-lane TMEM quarter; the
// 16-lane tcgen05.ld/st shapes spread those lanes over a whole warp: with
// .16x256b a thread holds rows r and r+8 of its quarter and key columns
// {8j + 2(t%4), 8j + 2(t%4) + 1}, so four threads share a row. P is packed to
// bf16 pairs and written back with .16x128b, whose column 4j + (t%4) is exactly
// the pair the thread holds. Softmax is online per row with lazy rescaling:
// the reference max of a row moves only when a score exceeds it by more than
// 2^8, after the first step of an item rarely.
//
// A tcgen05.mma issue occupies the issuing thread for about as long as an
// M=64 N=128 MMA runs, so the S and the O MMAs come from two issuing threads.
//
// Warp roles (512 threads):
//   warp 0      TMA producer of K (3-stage ring of steps)
//   warp 1      TMA producer of V (2-stage ring of steps)
//   warp 2      issuer of the S MMAs (also allocates tensor memory)
//   warp 3      issuer of the O MMAs
//   warps 4-11  softmax
//   warps 12-15 epilogue: Q copies (item is + 2 into the buffer of item is
//               as soon as item is's S products completed), gates and coarse
//               rows, output tiles (TMA)
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

constexpr int kThreads = 512;
constexpr int kKStages = 3;  // K ring depth (steps of two cubes)
constexpr int kVStages = 2;  // V ring depth
constexpr int kSP = 3;       // S/P buffers in tensor memory
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S/P buffer b at 128 b, O at 384.
constexpr uint32_t kColSP = 0, kColO = 384;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 3, 128;" ::: "memory"); }
// The two softmax warps of lane quarter q (warps 4+q and 8+q) use barrier 4+q.
__device__ __forceinline__ void pair_sync(int q) { asm volatile("bar.sync %0, 64;" ::"r"(4 + q) : "memory"); }
__device__ __forceinline__ bool pair_any(int q, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, o;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred o, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(4 + q)
      : "memory");
  return r != 0;
}

// Register split between warpgroups (the launch gives every thread 128):
// warps 0-3 (producers, MMA issuers) 72, softmax 152, epilogue 136;
// 128*72 + 256*152 + 128*136 = 65536 = 512*128: the increases (7168) are exactly
// what the decreases release, so they can always be met.
template <int N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// ---- 16-lane TMEM shapes (lanes base..base+15 of the warp's quarter) ----
#define VSA_O4(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3])
#define VSA_I4(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])
// .16x256b.x8: 64 columns; r[4j..4j+3] = (row a: col c, c+1; row a+8: col c, c+1), c = 8j + 2(t%4).
__device__ __forceinline__ void ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : VSA_O4(0), VSA_O4(4), VSA_O4(8), VSA_O4(12), VSA_O4(16), VSA_O4(20), VSA_O4(24), VSA_O4(28)
      : "r"(taddr));
}
__device__ __forceinline__ void st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12), VSA_I4(16), VSA_I4(20), VSA_I4(24), VSA_I4(28)
      : "memory");
}
// .16x128b.x8: 32 columns; r[2j] -> (row a, col 4j + t%4), r[2j+1] -> (row a+8, same col).
__device__ __forceinline__ void st_16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      VSA_I4(0), VSA_I4(4), VSA_I4(8), VSA_I4(12)
      : "memory");
}
#undef VSA_O4
#undef VSA_I4

// Softmax numerators of one 64-key half step for the thread's rows a and a+8
// (register layout of ld_16x256b_x8): P = 2^(s*scale - m), packed to bf16
// pairs (keys c, c+1 -> P column c/2), and the thread's partial row sums.
// All exponentials run on the MUFU pipe: moving a quarter of them to an FMA
// polynomial made the kernel 2% slower, since the FMA pipe already carries
// the scaling, the sums and the packing.
__device__ __forceinline__ void exp_pack(const uint32_t (&r)[32], float scale, float m0, float m1,
                                         uint32_t (&pk)[16], float& s0, float& s1) {
  const float nm0 = -m0, nm1 = -m1;
  s0 = 0.f;
  s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float x00 = fmaf(__uint_as_float(r[4 * j]), scale, nm0);
    const float x01 = fmaf(__uint_as_float(r[4 * j + 1]), scale, nm0);
    const float x10 = fmaf(__uint_as_float(r[4 * j + 2]), scale, nm1);
    const float x11 = fmaf(__uint_as_float(r[4 * j + 3]), scale, nm1);
    const float p00 = fast_exp2(x00);
    const float p01 = fast_exp2(x01);
    const float p10 = fast_exp2(x10);
    const float p11 = fast_exp2(x11);
    s0 += p00 + p01;
    s1 += p10 + p11;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(p00, p01);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(p10, p11);
    pk[2 * j] = *reinterpret_cast<uint32_t*>(&h0);
    pk[2 * j + 1] = *reinterpret_cast<uint32_t*>(&h1);
  }
}

// Unscaled maxima of rows a and a+8 over a 64-key half (the four threads of a
// row combine through shuffles).
__device__ __forceinline__ void half_row_max(const uint32_t (&r)[32], float& x0, float& x1) {
  float a[4], b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[j] = fmaxf(fmaxf(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])),
                 fmaxf(__uint_as_float(r[4 * j + 16]), __uint_as_float(r[4 * j + 17])));
    b[j] = fmaxf(fmaxf(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])),
                 fmaxf(__uint_as_float(r[4 * j + 18]), __uint_as_float(r[4 * j + 19])));
  }
  a[0] = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
  b[0] = fmaxf(fmaxf(b[0], b[1]), fmaxf(b[2], b[3]));
  x0 = fmaxf(a[0], __shfl_xor_sync(0xffffffffu, a[0], 1));
  x1 = fmaxf(b[0], __shfl_xor_sync(0xffffffffu, b[0], 1));
  x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
  x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
}

template <int D>
struct Layout {
  static constexpr int NH = D / 64;              // 128-byte column groups of a row
  static constexpr int Q_BYTES = 64 * D * 2;     // one query cube
  static constexpr int KV_BYTES = 128 * D * 2;   // two KV cubes
  static constexpr int OFF_Q = 0;                                 // Q[2]
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;               // K ring
  static constexpr int OFF_V = OFF_K + kKStages * KV_BYTES;       // V ring
  static constexpr int OFF_STAGE = OFF_V + kVStages * KV_BYTES;   // output staging, 64 x D bf16
  static constexpr int TILE_BYTES = OFF_STAGE + 64 * D * 2;
  static constexpr int SMEM_BYTES = TILE_BYTES + 1024;            // + alignment slack
};

struct __align__(8) Bars {
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t q_full[2];     // Q of item is in smem buffer is % 2 (count 128: every epilogue thread)
  uint64_t q_free[2];     // S issuer -> epilogue: every S product of item is complete (commit)
  uint64_t lp_free[2];    // epilogue -> softmax: row statistics of item is read (count 4)
  uint64_t s_full[kSP];   // S issuer -> softmax: S of step j in buffer j % 3 (commit)
  uint64_t p_full[kSP];   // softmax -> O issuer: P of step j in buffer j % 3 (count 8)
  uint64_t sp_free[kSP];  // O issuer -> S issuer, softmax: O of step j complete (commit)
  uint64_t l_full[2];     // softmax -> epilogue: row sums of item is in lpart[is % 2] (count 8)
  uint64_t o_full;        // O issuer -> epilogue: O of an item complete (commit)
  uint64_t o_empty;       // epilogue -> O issuer: O read out (count 4)
  uint64_t drain[2], stall;
};

// Gates and coarse output of one item, prefetched by the epilogue.
struct alignas(16) Pre {
  float gc[64], gf[64];  // per in-cube slot
  float oc[128];         // coarse output row (D values)
};

struct alignas(16) Shared {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float xmax[2][64];      // [key half][row]: half-row maxima on the rescale path
  alignas(16) float lpart[2][2][64];  // [item parity][key half][row]: row sums of an item
  alignas(16) float mref[2][64];      // [item parity][row]: final reference max (log2 units) of an item
  Pre pre[2];                         // [item parity]
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

// The item at the CTA's position `is`, or -1 past the end. Without an order
// array the CTA takes items blockIdx.x + is * gridDim.x; with one (variable
// counts) it takes the positions of a serpentine hand-out of the array,
// which lists each head's items longest first (schedule.cu).
__device__ __forceinline__ int item_at(const FineParams& p, int is) {
  const int G = gridDim.x, c = blockIdx.x;
  const int pos = is * G + ((p.order && (is & 1)) ? G - 1 - c : c);
  if (pos >= p.n_items) return -1;
  return p.order ? p.order[pos] : pos;
}

// Selected-cube count of an item as stored (validated when the item is reached).
__device__ __forceinline__ int raw_count(const FineParams& p, int item) {
  if (item < 0) return 0;
  return p.cnt ? p.cnt[item] : p.kcap;
}

// Position in the CTA's sequence of steps (items item_at(p, is)).
// The count of the next item is loaded one item ahead, so no role stalls on
// it at an item boundary.
struct Cursor {
  int is;      // item index within the CTA
  int item;    // global item index
  int n;       // selected cubes of the item
  int n_next;  // raw count of the next item
  int t;       // step within the item
  int ntiles;  // steps of the item
  bool live;
  bool bad;    // a count outside [1, kcap] was seen (and clamped)
};
__device__ __forceinline__ void cursor_enter(const FineParams& p, Cursor& c, int n_raw) {
  c.live = c.item >= 0;
  int n = n_raw;
  if (c.live && (n < 1 || n > p.kcap)) {
    c.bad = true;
    n = n < 1 ? 1 : p.kcap;
  }
  c.n = c.live ? n : 0;
  c.t = 0;
  c.ntiles = (c.n + 1) >> 1;
}
__device__ __forceinline__ void cursor_init(const FineParams& p, Cursor& c) {
  c.is = 0;
  c.item = item_at(p, 0);
  c.bad = false;
  const int n0 = raw_count(p, c.item);
  c.n_next = raw_count(p, item_at(p, 1));
  cursor_enter(p, c, n0);
}
__device__ __forceinline__ void cursor_next(const FineParams& p, Cursor& c) {
  if (++c.t < c.ntiles) return;
  c.is += 1;
  c.item = item_at(p, c.is);
  const int n_raw = c.n_next;
  c.n_next = raw_count(p, item_at(p, c.is + 1));
  cursor_enter(p, c, n_raw);
}

// Rows a and a+8 of a 64-column O block scaled by a0 and a1 (one warp).
__device__ __forceinline__ void rescale_o64(uint32_t taddr, float a0, float a1) {
  uint32_t o[32];
  ld_16x256b_x8(taddr, o);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o[4 * e] = __float_as_uint(__uint_as_float(o[4 * e]) * a0);
    o[4 * e + 1] = __float_as_uint(__uint_as_float(o[4 * e + 1]) * a0);
    o[4 * e + 2] = __float_as_uint(__uint_as_float(o[4 * e + 2]) * a1);
    o[4 * e + 3] = __float_as_uint(__uint_as_float(o[4 * e + 3]) * a1);
  }
  st_16x256b_x8(taddr, o);
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
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&B.k_full[i], 1);
      mbar_init(&B.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&B.v_full[i], 1);
      mbar_init(&B.v_empty[i], 1);
    }
    for (int b = 0; b < kSP; ++b) {
      mbar_init(&B.s_full[b], 1);
      mbar_init(&B.p_full[b], 8);
      mbar_init(&B.sp_free[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.q_full[b], 128);
      mbar_init(&B.l_full[b], 8);
      mbar_init(&B.drain[b], 1);
      mbar_init(&B.q_free[b], 1);
      mbar_init(&B.lp_free[b], 4);
    }
    mbar_init(&B.o_full, 1);
    mbar_init(&B.o_empty, 4);
    mbar_init(&B.stall, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    if (p.out) prefetch_tmap(&p.tm_out);
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
    // ------------------------------------------------------------ K (warp 0) / V (warp 1) producer
    regs_dec<72>();
    const bool is_k = (warp == 0);
    const int stages = is_k ? kKStages : kVStages;
    uint64_t* full = is_k ? B.k_full : B.v_full;
    uint64_t* empty = is_k ? B.k_empty : B.v_empty;
    uint8_t* ring = tiles + (is_k ? L::OFF_K : L::OFF_V);
    const CUtensorMap* tm = is_k ? &p.tm_k : &p.tm_v;
    bool bad = false, aborted = false;
    int g = 0;  // steps armed
    // Cube ids of a step: lanes 0 and 1 load them; -1 if absent.
    auto fetch = [&](const Cursor& c) -> int {
      int cid = -1;
      if (lane < 2 && c.live) {
        const int e = 2 * c.t + lane;
        if (e < c.n) cid = p.idx[(size_t)c.item * p.kcap + e];
      }
      return cid;
    };
    Cursor c;
    cursor_init(p, c);
    int cid = fetch(c);
    while (c.live) {
      Cursor nx = c;  // look one step ahead so the id loads overlap this step
      cursor_next(p, nx);
      const int cid_next = fetch(nx);
      int ca = __shfl_sync(0xffffffffu, cid, 0);
      int cb = __shfl_sync(0xffffffffu, cid, 1);
      if (cb < 0) cb = ca;  // odd tail: load a copy, the softmax masks it
      if (ca < 0 || ca >= C || cb < 0 || cb >= C) {
        bad = true;
        ca = ca < 0 || ca >= C ? 0 : ca;
        cb = cb < 0 || cb >= C ? 0 : cb;
      }
      const int bh = c.item / C;
      if (lane == 0) {
        const int slot = g % stages;
        if (g >= stages && !W.wait(&empty[slot], ((g / stages) - 1) & 1)) aborted = true;
        if (!aborted) {
          mbar_arrive_expect_tx(&full[slot], L::KV_BYTES);
          uint8_t* dst = ring + slot * L::KV_BYTES;
#pragma unroll
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(dst + h * 16384, tm, &full[slot], 64 * h, (bh * C + ca) * 64);
            tma_load_2d(dst + h * 16384 + 8192, tm, &full[slot], 64 * h, (bh * C + cb) * 64);
          }
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
      if (aborted) break;
      ++g;
      c = nx;
      cid = cid_next;
    }
    if (is_k && (bad || c.bad) && lane == 0) atomicOr(p.err, kErrBadIndex);
    // Drain: phases complete in order, so waiting for the last armed phase of
    // each slot covers every copy this warp issued.
    if (lane == 0)
      for (int slot = 0; slot < stages && slot < g; ++slot) {
        const int uses = (g - 1 - slot) / stages + 1;
        W.drain_wait(&full[slot], (uses - 1) & 1);
      }
  } else if (warp == 2) {
    // ------------------------------------------------------------ S issuer
    regs_dec<72>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(64, 128, false, false);
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_Q), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_K), 16, 1024);
      bool aborted = false, issued_any = false;
      if (p.debug_stall && !W.wait(&B.stall, 0)) aborted = true;
      Cursor c;
      cursor_init(p, c);
      int j = 0;         // steps of the CTA
      int b = 0, u = 0;  // S/P buffer of step j (j % 3) and its use count (j / 3)
      while (!aborted && c.live) {
        const int ks = j % kKStages;
        // Buffer b is free once O of step j - 3 (which read its P) completed.
        if ((u >= 1 && !W.wait(&B.sp_free[b], (u - 1) & 1)) ||
            (c.t == 0 && !W.wait(&B.q_full[c.is & 1], (c.is >> 1) & 1)) ||
            !W.wait(&B.k_full[ks], (j / kKStages) & 1)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint64_t qd = qdesc0 + (uint64_t)(((c.is & 1) * L::Q_BYTES) >> 4);
        const uint64_t kd = kdesc0 + (uint64_t)((ks * L::KV_BYTES) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)  // steps of 16 along D
          mma_bf16_ss(tmem + kColSP + 128u * b, qd + (uint64_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4),
                      kd + (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4), idesc_s, k > 0 ? 1u : 0u);
        mma_commit(&B.k_empty[ks]);
        mma_commit(&B.s_full[b]);
        // The item's last S product: once it completes, its Q buffer is free.
        if (c.t == c.ntiles - 1) mma_commit(&B.q_free[c.is & 1]);
        issued_any = true;
        ++j;
        if (++b == kSP) { b = 0; ++u; }
        cursor_next(p, c);
      }
      // Drain: every MMA issued by this thread completes before TMEM is released.
      if (issued_any) {
        mma_commit(&B.drain[0]);
        W.drain_wait(&B.drain[0], 0);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ O issuer
    regs_dec<72>();
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16_f32(64, D, false, true);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_V), 16384, 1024);
      bool aborted = false, issued_any = false;
      Cursor c;
      cursor_init(p, c);
      int j = 0;
      int b = 0, u = 0;  // S/P buffer of step j and its use count
      while (!aborted && c.live) {
        const int vs = j % kVStages;
        const bool first = (c.t == 0), last = (c.t == c.ntiles - 1);
        if ((first && c.is >= 1 && !W.wait(&B.o_empty, (c.is - 1) & 1)) ||
            !W.wait(&B.v_full[vs], (j / kVStages) & 1) || !W.wait(&B.p_full[b], u & 1)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint64_t vd = vdesc0 + (uint64_t)((vs * L::KV_BYTES) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 8 steps of 16 keys; P step k = 8 TMEM columns
          mma_bf16_ts(tmem + kColO, tmem + kColSP + 128u * b + 8u * k, vd + (uint64_t)((k * 2048) >> 4), idesc_o,
                      (first && k == 0) ? 0u : 1u);
        mma_commit(&B.v_empty[vs]);
        mma_commit(&B.sp_free[b]);
        if (last) mma_commit(&B.o_full);
        issued_any = true;
        ++j;
        if (++b == kSP) { b = 0; ++u; }
        cursor_next(p, c);
      }
      if (issued_any) {
        mma_commit(&B.drain[1]);
        W.drain_wait(&B.drain[1], 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax
    regs_inc<152>();
    const int quarter = warp & 3, hf = (warp - 4) >> 2;  // lane quarter, key half
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);  // rows ra and ra + 8
    const float scale = p.scale_log2;
    int b = 0, u = 0;  // S/P buffer of the step (step % 3) and its use count (step / 3)
    Cursor c;
    cursor_init(p, c);
    while (c.live) {
      const int n = c.n, ntiles = c.ntiles, ob = c.is & 1;
      float m0 = -INFINITY, m1 = -INFINITY;  // reference max (scaled) of rows ra and ra+8
      float l0 = 0.f, l1 = 0.f;              // this thread's share of the row sums
      for (int t = 0; t < ntiles; ++t) {
        const uint32_t tS = tmem + kColSP + 128u * b + lane_base;
        W.wait(&B.s_full[b], u & 1);
        tc_fence_after();
        uint32_t r[32];
        ld_16x256b_x8(tS + 64u * hf, r);
        tmem_wait_ld();
        // Odd tail: keys 64..127 (the repeated cube) do not take part.
        const bool masked = hf == 1 && (2 * t + 1 >= n);
        if (masked) {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(-INFINITY);
        }
        // Optimistic pass with the current reference max. A thread's partial
        // row sum exceeds 2^8 whenever one of its scores exceeds the reference
        // by more than 2^8, so only then are the exact row maxima needed. The
        // first step of an item (reference still -inf) goes there directly.
        uint32_t pk[16];
        float s0 = 0.f, s1 = 0.f;
        bool exact = true;
        if (t > 0) {
          exp_pack(r, scale, m0, m1, pk, s0, s1);
          exact = pair_any(quarter, !(s0 <= 256.f) || !(s1 <= 256.f));
        }
        if (exact) {
          float x0, x1;
          half_row_max(r, x0, x1);
          if ((lane & 3) == 0) {
            sh.xmax[hf][ra] = x0;
            sh.xmax[hf][ra + 8] = x1;
          }
          pair_sync(quarter);
          x0 = fmaxf(sh.xmax[0][ra], sh.xmax[1][ra]) * scale;
          x1 = fmaxf(sh.xmax[0][ra + 8], sh.xmax[1][ra + 8]) * scale;
          pair_sync(quarter);
          // Lazy reference update per row (identical in both warps of the pair).
          float a0 = 1.f, a1 = 1.f;
          const bool u0 = x0 > m0 + 8.0f, u1 = x1 > m1 + 8.0f;
          if (u0) { a0 = fast_exp2(m0 - x0); m0 = x0; l0 *= a0; }
          if (u1) { a1 = fast_exp2(m1 - x1); m1 = x1; l1 *= a1; }
          if (__any_sync(0xffffffffu, u0 || u1)) {
            if (t > 0 && (D == 128 || hf == 0)) {
              // O holds steps < t of this item: wait for the last of them to
              // complete, then rescale this warp's 64 columns of the rows
              // (D = 64: the first warp of the pair takes all of them).
              const int pb = b == 0 ? kSP - 1 : b - 1, pu = b == 0 ? u - 1 : u;  // buffer, use of step - 1
              W.wait(&B.sp_free[pb], pu & 1);
              tc_fence_after();
              rescale_o64(tmem + kColO + lane_base + (D == 128 ? 64u * hf : 0u), a0, a1);
              tmem_wait_st();
            }
            exp_pack(r, scale, m0, m1, pk, s0, s1);
          }
        }
        l0 += s0;
        l1 += s1;
        st_16x128b_x8(tS + 32u * hf, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[b]);
        if (++b == kSP) { b = 0; ++u; }
      }
      // Row sums of the item (this key half) -> the epilogue, once it has read
      // those of the item two back (the same entries).
      if (c.is >= 2) W.wait(&B.lp_free[ob], ((c.is >> 1) - 1) & 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if ((lane & 3) == 0) {
        sh.lpart[ob][hf][ra] = l0;
        sh.lpart[ob][hf][ra + 8] = l1;
        if (hf == 0) {
          sh.mref[ob][ra] = m0;
          sh.mref[ob][ra + 8] = m1;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.l_full[ob]);
      c.t = c.ntiles - 1;
      cursor_next(p, c);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue (+ Q loads)
    regs_inc<136>();
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int ra = quarter * 16 + (lane >> 2);  // rows ra and ra + 8 of the item
    const int tq = lane & 3;
    const int est = tid - 384;                  // 0..127 within the epilogue group
    uint8_t* stage = tiles + L::OFF_STAGE;
    const int Hc = p.H >> 2, Wc = p.W >> 2;
    int qloads0 = 0, qloads1 = 0;
    // Q of item `is` -> smem buffer is & 1: each epilogue thread copies 16-byte
    // chunks of token rows (cp.async) to chunk c ^ (row % 8) of the row, the
    // 128-byte swizzle of the MMA operand; the copies complete in the thread's
    // cp.async group and are published by q_arrive (proxy fence, then one
    // arrival per thread on q_full).
    constexpr int CPR = D / 8, RPI = 128 / CPR;  // 16-byte chunks per token row, rows per pass
    auto load_q = [&](int is) {
      const int item = item_at(p, is);
      if (item < 0) return;
      const int b = is & 1;
      if (b == 0) ++qloads0; else ++qloads1;
      const int bh = item / C, ci = item - bh * C;
      const int ct = ci / (Hc * Wc), ch = (ci / Wc) % Hc, cw = ci % Wc;
      uint8_t* dst = tiles + L::OFF_Q + b * L::Q_BYTES;
      const int chunk = est % CPR, r0 = est / CPR, h = chunk >> 3, cc = chunk & 7;
#pragma unroll
      for (int i = 0; i < 64 / RPI; ++i) {
        const int r = r0 + RPI * i;
        const int tok = ((4 * ct + (r >> 4)) * p.H + 4 * ch + ((r >> 2) & 3)) * p.W + 4 * cw + (r & 3);
        cp_async16(dst + h * 8192 + r * 128 + ((cc ^ (r & 7)) << 4), p.q + ((size_t)bh * p.N + tok) * D + chunk * 8);
      }
    };
    auto q_arrive = [&](int is) {
      if (item_at(p, is) < 0) return;
      fence_proxy_async_smem();
      mbar_arrive(&B.q_full[is & 1]);
    };
    // Gates (16 runs of 4 raster tokens per gate array) and the coarse output
    // row of item `is` -> sh.pre[is & 1]; one cp.async group per call on
    // every thread, so groups stay in the same order everywhere.
    auto prefetch = [&](int is) {
      const int item = item_at(p, is);
      if (item >= 0 && est < 32 + D / 4) {
        const int bh = item / C, ci = item - bh * C;
        Pre& pr = sh.pre[is & 1];
        if (est < 32) {
          const int run = est & 15;  // in-cube slots 4 run .. 4 run + 3: t = run / 4, h = run % 4
          const int ct = ci / (Hc * Wc), ch = (ci / Wc) % Hc, cw = ci % Wc;
          const int tok = ((4 * ct + (run >> 2)) * p.H + 4 * ch + (run & 3)) * p.W + 4 * cw;
          const float* g = (est < 16 ? p.gate_c : p.gate_f) + (size_t)bh * p.N + tok;
          cp_async16(est < 16 ? &pr.gc[4 * run] : &pr.gf[4 * run], g);
        } else {
          const int e = est - 32;
          cp_async16(&pr.oc[4 * e], p.oc + ((size_t)bh * C + ci) * D + 4 * e);
        }
      }
      cp_async_commit();
    };
    load_q(0);
    load_q(1);
    cp_async_commit();
    prefetch(0);
    cp_async_wait<1>();
    q_arrive(0);
    q_arrive(1);
    for (int is = 0; item_at(p, is) >= 0; ++is) {
      const int item = item_at(p, is);
      const int bh = item / C, ci = item - bh * C;
      const int ct = ci / (Hc * Wc), ch = (ci / Wc) % Hc, cw = ci % Wc;
      const int ob = is & 1;
      // Q of item is + 2 goes into this item's buffer as soon as the item's
      // S products have completed, not after its O read-out, so the copies
      // from HBM have most of an item to land (waiting for the O read-out
      // left the S issuer stalled on Q at item boundaries).
      const bool qnext = item_at(p, is + 2) >= 0 && W.wait(&B.q_free[ob], (is >> 1) & 1);
      if (qnext) load_q(is + 2);
      cp_async_commit();
      prefetch(is + 1);
      W.wait(&B.l_full[ob], (is >> 1) & 1);
      const float lsum0 = sh.lpart[ob][0][ra] + sh.lpart[ob][1][ra];
      const float lsum1 = sh.lpart[ob][0][ra + 8] + sh.lpart[ob][1][ra + 8];
      const float il0 = 1.0f / lsum0, il1 = 1.0f / lsum1;
      // raster token of in-cube slot q: ((4ct + q/16) H + 4ch + (q/4)%4) W + 4cw + q%4
      auto tok_of = [&](int q) { return ((4 * ct + (q >> 4)) * p.H + 4 * ch + ((q >> 2) & 3)) * p.W + 4 * cw + (q & 3); };
      if (p.lse && tq == 0) {
        // natural log of the row's denominator: ln 2 * (reference max + log2 of the sum)
        p.lse[(size_t)bh * p.N + tok_of(ra)] = 0.6931471805599453f * (sh.mref[ob][ra] + __log2f(lsum0));
        p.lse[(size_t)bh * p.N + tok_of(ra + 8)] = 0.6931471805599453f * (sh.mref[ob][ra + 8] + __log2f(lsum1));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.lp_free[ob]);  // row statistics of item is read
      W.wait(&B.o_full, is & 1);
      tc_fence_after();
      float o[2 * D / 4];
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t r[32];
        ld_16x256b_x8(tmem + kColO + 64u * h + lane_base, r);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) o[32 * h + jj] = __uint_as_float(r[jj]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.o_empty);
      cp_async_wait<1>();               // this item's gates and coarse row (older group) landed
      if (qnext) q_arrive(is + 2);
      if (est == 0) bulk_wait_read0();  // the previous item's output stores have read the staging tile
      epi_sync();
      const Pre& pr = sh.pre[ob];
      const float gc0 = pr.gc[ra], gf0 = pr.gf[ra], gc1 = pr.gc[ra + 8], gf1 = pr.gf[ra + 8];
      // o[4j..4j+3] = (row ra: d, d+1; row ra+8: d, d+1), d = 8j + 2 tq
      if (p.o_fine) {
        const int tok0 = tok_of(ra), tok1 = tok_of(ra + 8);
#pragma unroll
        for (int jj = 0; jj < D / 8; ++jj) {
          const int d = 8 * jj + 2 * tq;
          *reinterpret_cast<float2*>(p.o_fine + ((size_t)bh * p.N + tok0) * D + d) =
              make_float2(o[4 * jj] * il0, o[4 * jj + 1] * il0);
          *reinterpret_cast<float2*>(p.o_fine + ((size_t)bh * p.N + tok1) * D + d) =
              make_float2(o[4 * jj + 2] * il1, o[4 * jj + 3] * il1);
        }
      }
      if (p.out_fine) {
        const int tok0 = tok_of(ra), tok1 = tok_of(ra + 8);
#pragma unroll
        for (int jj = 0; jj < D / 8; ++jj) {
          const int d = 8 * jj + 2 * tq;
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok0) * D + d) =
              make_float2(o[4 * jj] * il0, o[4 * jj + 1] * il0);
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok1) * D + d) =
              make_float2(o[4 * jj + 2] * il1, o[4 * jj + 3] * il1);
        }
      }
      if (p.out) {
        // Staging tile: per 64-column group a [64 slots][128 B] block in the
        // 128-byte swizzle of the output map (16-byte chunk c of row q at
        // c ^ (q % 8)); rows ra and ra + 8 share q % 8.
        const float f0 = gf0 * il0, f1 = gf1 * il1;
        const uint32_t sw = (uint32_t)(ra & 7);
#pragma unroll
        for (int jj = 0; jj < D / 8; ++jj) {
          const int d = 8 * jj + 2 * tq;
          const float2 oc = *reinterpret_cast<const float2*>(&pr.oc[d]);
          const __nv_bfloat162 h0 =
              __floats2bfloat162_rn(fmaf(gc0, oc.x, f0 * o[4 * jj]), fmaf(gc0, oc.y, f0 * o[4 * jj + 1]));
          const __nv_bfloat162 h1 =
              __floats2bfloat162_rn(fmaf(gc1, oc.x, f1 * o[4 * jj + 2]), fmaf(gc1, oc.y, f1 * o[4 * jj + 3]));
          uint8_t* blk = stage + (jj >> 3) * 8192 + ((((uint32_t)jj & 7u) ^ sw) << 4) + 4 * tq;
          *reinterpret_cast<__nv_bfloat162*>(blk + ra * 128) = h0;
          *reinterpret_cast<__nv_bfloat162*>(blk + (ra + 8) * 128) = h1;
        }
        fence_proxy_async_smem();
        epi_sync();
        if (est == 0) {
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_store_5d(&p.tm_out, stage + h * 8192, 64 * h, 4 * cw, 4 * ch, 4 * ct, bh);
          bulk_commit();
        }
      } else {
        epi_sync();  // this item's gate reads are done before the buffer refills
      }
    }
    cp_async_wait<0>();
    // Drain: the output stores are complete and the last Q copy of each
    // buffer has landed (it has, unless the run aborted).
    if (est == 0) {
      bulk_wait0();
      if (qloads0 > 0) W.drain_wait(&B.q_full[0], (qloads0 - 1) & 1);
      if (qloads1 > 0) W.drain_wait(&B.q_full[1], (qloads1 - 1) & 1);
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
