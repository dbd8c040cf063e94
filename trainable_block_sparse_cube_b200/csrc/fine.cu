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
//
// Two item streams run interleaved (the CTA's even and odd items), each with
// its own TMA producer warp, K and V buffers, MMA-issuing warp, softmax
// warpgroup, S/P buffer and O accumulator in tensor memory, so the tensor core
// always has the other stream's work while one stream's softmax runs. The
// streams share nothing but the tensor core and the epilogue: each issuer
// keeps its own stream's order [S(0)], [O(j), S(j+1)], ... . A tcgen05.mma
// issue occupies the issuing thread for about as long as an M=64 N=128 MMA
// runs, so a single issuing thread leaves no slack for its waits; one issuing
// thread per stream keeps the tensor core fed while the other one waits.
// Because a tcgen05 commit covers every earlier MMA of the issuing thread,
// "S(j+1) complete" also means "O(j) complete": when a softmax warp sees its
// next S it may overwrite P in place and rescale O.
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
// Warp roles (512 threads):
//   warps 0, 1  TMA producer of stream 0, 1: K and V of a step (one buffer
//               each; two issuing threads keep the L2 -> SM stream full)
//   warps 2, 3  single-thread tcgen05.mma issuer of stream 0, 1 (warp 2 also
//               allocates tensor memory)
//   warps 4-7   softmax of stream 0     warps 8-11  softmax of stream 1
//   warps 12-15 epilogue: Q loads, 1/l and gates, output rows
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
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S/P of stream s at 128 s, O of stream s at 256 + 128 s.
constexpr uint32_t kColSP = 0, kColO = 256;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 3, 128;" ::: "memory"); }

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
// .16x256b.x8: 64 columns, 32 registers.
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

// 2^x on the FMA pipe, for x in [-126, 64] (clamped): x = n + f with n the
// nearest integer (added to 1.5 * 2^23 so that it lands in the low mantissa
// bits) and f in [-1/2, 1/2]; 2^f is a cubic fitted by weighted least squares
// (relative error) on Chebyshev nodes of [-1/2, 1/2], max relative error
// 7.8e-5, far below the bf16 rounding of P; 2^n is added to the exponent
// field. Offloads part of the exponentials from the 16-per-clock MUFU units.
__device__ __forceinline__ float poly_exp2(float x) {
  x = fminf(fmaxf(x, -126.f), 64.f);
  const float t = __fadd_rn(x, 12582912.f);
  const float f = __fsub_rn(x, __fsub_rn(t, 12582912.f));
  float p = fmaf(0.05508868396282196f, f, 0.24260404706001282f);
  p = fmaf(p, f, 0.6932762265205383f);
  p = fmaf(p, f, 0.9999289512634277f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Softmax numerators of one 128-key step for the thread's rows a and a+8
// (register layout of ld_16x256b_x16): P = 2^(s*scale - m), packed to bf16
// pairs (keys c, c+1 -> P column c/2), and the thread's partial row sums.
// With POLY one column group in four takes the FMA-pipe exponential; masked
// (-inf) scores need the exact zero of the MUFU path.
template <bool POLY>
__device__ __forceinline__ void exp_pack(const uint32_t (&r)[64], float scale, float m0, float m1,
                                         uint32_t (&pk)[32], float& s0, float& s1) {
  const float nm0 = -m0, nm1 = -m1;
  s0 = 0.f;
  s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const bool poly = POLY && (j & 3) == 3;
    const float x00 = fmaf(__uint_as_float(r[4 * j]), scale, nm0);
    const float x01 = fmaf(__uint_as_float(r[4 * j + 1]), scale, nm0);
    const float x10 = fmaf(__uint_as_float(r[4 * j + 2]), scale, nm1);
    const float x11 = fmaf(__uint_as_float(r[4 * j + 3]), scale, nm1);
    const float p00 = poly ? poly_exp2(x00) : fast_exp2(x00);
    const float p01 = poly ? poly_exp2(x01) : fast_exp2(x01);
    const float p10 = poly ? poly_exp2(x10) : fast_exp2(x10);
    const float p11 = poly ? poly_exp2(x11) : fast_exp2(x11);
    s0 += p00 + p01;
    s1 += p10 + p11;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(p00, p01);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(p10, p11);
    pk[2 * j] = *reinterpret_cast<uint32_t*>(&h0);
    pk[2 * j + 1] = *reinterpret_cast<uint32_t*>(&h1);
  }
}

// Unscaled maxima of rows a and a+8 over the whole 128-key step (the four
// threads of a row combine through shuffles).
__device__ __forceinline__ void row_max(const uint32_t (&r)[64], float& x0, float& x1) {
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    a[j] = fmaxf(fmaxf(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])),
                 fmaxf(__uint_as_float(r[4 * j + 32]), __uint_as_float(r[4 * j + 33])));
    b[j] = fmaxf(fmaxf(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])),
                 fmaxf(__uint_as_float(r[4 * j + 34]), __uint_as_float(r[4 * j + 35])));
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; ++j) {
      a[j] = fmaxf(a[j], a[j + w]);
      b[j] = fmaxf(b[j], b[j + w]);
    }
  x0 = fmaxf(a[0], __shfl_xor_sync(0xffffffffu, a[0], 1));
  x1 = fmaxf(b[0], __shfl_xor_sync(0xffffffffu, b[0], 1));
  x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
  x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
}

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
  static constexpr int Q_BYTES = 64 * D * 2;     // one query cube
  static constexpr int KV_BYTES = 128 * D * 2;   // two KV cubes
  static constexpr int OFF_Q = 0;                                 // Q[stream][2]
  static constexpr int OFF_K = OFF_Q + 4 * Q_BYTES;               // K[stream]
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;              // V[stream]
  static constexpr int OFF_STAGE = OFF_V + 2 * KV_BYTES;          // output staging, 64 x D bf16
  static constexpr int TILE_BYTES = OFF_STAGE + 64 * D * 2;
  static constexpr int SMEM_BYTES = TILE_BYTES + 1024;            // + alignment slack
};

struct __align__(8) Bars {
  uint64_t k_full[2], k_empty[2];  // [stream]: K of a step in smem / consumed
  uint64_t v_full[2], v_empty[2];  // [stream]: V of a step in smem / consumed
  uint64_t q_full[2][2];   // [stream][buffer]: Q of an item in smem (TMA)
  uint64_t s_full[2];      // MMA -> softmax of stream s: S of a step (commit)
  uint64_t p_full[2];      // softmax -> MMA: P of a step in TMEM (count 4)
  uint64_t l_full[2][2];   // softmax -> epilogue: 1/l of an item (count 4)
  uint64_t o_full[2];      // MMA -> epilogue: last O step of an item (commit)
  uint64_t o_empty[2];     // epilogue -> MMA: O read out (count 4)
  uint64_t drain[2], stall;
};

struct alignas(16) Shared {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  int issue_lock;                     // held by an MMA issuer while it enqueues a block
  int epi_pick;                       // stream whose item the epilogue handles next
  alignas(16) float inv_l[2][2][64];  // [stream][item parity][row]
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
  // Bounded acquisition of a shared-memory spin lock; false on timeout or abort.
  __device__ __forceinline__ bool acquire(int* lock) const {
    if (atomicCAS(lock, 0, 1) == 0) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 64; ++i)
        if (atomicCAS(lock, 0, 1) == 0) return true;
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

// Selected-cube count of an item as stored (validated when the item is reached).
__device__ __forceinline__ int raw_count(const FineParams& p, int item) {
  if (item >= p.n_items) return 0;
  return p.cnt ? p.cnt[item] : p.kcap;
}

// Position of one stream in its own sequence of steps. The count of the
// stream's next item is loaded one item ahead, so no role stalls on it at an
// item boundary.
struct Cursor {
  int is;      // item index within the stream
  int item;    // global item index
  int n;       // selected cubes of the item
  int n_next;  // raw count of the stream's next item
  int t;       // step within the item
  int ntiles;  // steps of the item
  bool live;
  bool bad;    // a count outside [1, kcap] was seen (and clamped)
};
__device__ __forceinline__ void cursor_enter(const FineParams& p, Cursor& c, int n_raw) {
  c.live = c.item < p.n_items;
  int n = n_raw;
  if (c.live && (n < 1 || n > p.kcap)) {
    c.bad = true;
    n = n < 1 ? 1 : p.kcap;
  }
  c.n = c.live ? n : 0;
  c.t = 0;
  c.ntiles = (c.n + 1) >> 1;
}
__device__ __forceinline__ void cursor_init(const FineParams& p, Cursor& c, int s) {
  c.is = 0;
  c.item = blockIdx.x + s * gridDim.x;
  c.bad = false;
  const int n0 = raw_count(p, c.item);
  c.n_next = raw_count(p, c.item + 2 * gridDim.x);
  cursor_enter(p, c, n0);
}
__device__ __forceinline__ void cursor_next(const FineParams& p, Cursor& c) {
  if (++c.t < c.ntiles) return;
  c.is += 1;
  c.item += 2 * gridDim.x;
  const int n_raw = c.n_next;
  c.n_next = raw_count(p, c.item + 2 * gridDim.x);
  cursor_enter(p, c, n_raw);
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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.k_empty[s], 1);
      mbar_init(&B.v_full[s], 1);
      mbar_init(&B.v_empty[s], 1);
      mbar_init(&B.drain[s], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&B.q_full[s][b], 1);
        mbar_init(&B.l_full[s][b], 4);
      }
      mbar_init(&B.s_full[s], 1);
      mbar_init(&B.p_full[s], 4);
      mbar_init(&B.o_full[s], 1);
      mbar_init(&B.o_empty[s], 4);
    }
    mbar_init(&B.stall, 1);
    sh.abort_flag = 0;
    sh.issue_lock = 0;
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

  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------ K / V producer of stream s
    regs_dec<72>();
    const int s = warp;
    uint8_t* kbuf = tiles + L::OFF_K + s * L::KV_BYTES;
    uint8_t* vbuf = tiles + L::OFF_V + s * L::KV_BYTES;
    bool bad = false, aborted = false;
    int g = 0;                   // steps issued
    int k_armed = 0, v_armed = 0;  // copies armed on k_full / v_full (lane 0)
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
    cursor_init(p, c, s);
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
      const int row_a = (c.item / C * C + ca) * 64, row_b = (c.item / C * C + cb) * 64;
      if (lane == 0) {
        if (g >= 1 && !W.wait(&B.k_empty[s], (g - 1) & 1)) aborted = true;
        if (!aborted) {
          mbar_arrive_expect_tx(&B.k_full[s], L::KV_BYTES);
          ++k_armed;
#pragma unroll
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(kbuf + h * 16384, &p.tm_k, &B.k_full[s], 64 * h, row_a);
            tma_load_2d(kbuf + h * 16384 + 8192, &p.tm_k, &B.k_full[s], 64 * h, row_b);
          }
        }
        if (!aborted && g >= 1 && !W.wait(&B.v_empty[s], (g - 1) & 1)) aborted = true;
        if (!aborted) {
          mbar_arrive_expect_tx(&B.v_full[s], L::KV_BYTES);
          ++v_armed;
#pragma unroll
          for (int h = 0; h < L::NH; ++h) {
            tma_load_2d(vbuf + h * 16384, &p.tm_v, &B.v_full[s], 64 * h, row_a);
            tma_load_2d(vbuf + h * 16384 + 8192, &p.tm_v, &B.v_full[s], 64 * h, row_b);
          }
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
      if (aborted) break;
      ++g;
      c = nx;
      cid = cid_next;
    }
    if ((bad || c.bad) && lane == 0) atomicOr(p.err, kErrBadIndex);
    // Drain: phases complete in order, so waiting for the last armed phase of
    // each barrier covers every copy this warp issued.
    if (lane == 0 && k_armed > 0) W.drain_wait(&B.k_full[s], (k_armed - 1) & 1);
    if (lane == 0 && v_armed > 0) W.drain_wait(&B.v_full[s], (v_armed - 1) & 1);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ MMA issuer of stream s
    regs_dec<72>();
    if (lane == 0) {
      const int s = warp - 2;
      constexpr uint32_t idesc_s = idesc_bf16_f32(64, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(64, D, false, true);
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(tiles + L::OFF_Q + 2 * s * L::Q_BYTES), 16, 1024);
      const uint64_t kdesc = sdesc_sw128(smem_u32(tiles + L::OFF_K + s * L::KV_BYTES), 16, 1024);
      const uint64_t vdesc = sdesc_sw128(smem_u32(tiles + L::OFF_V + s * L::KV_BYTES), 16384, 1024);
      const uint32_t tS = tmem + kColSP + 128u * s, tO = tmem + kColO + 128u * s;
      bool aborted = false, issued_any = false;
      if (p.debug_stall && !W.wait(&B.stall, 0)) aborted = true;
      Cursor c;
      cursor_init(p, c, s);
      int j = 0;  // steps of this stream
      // Each block ([S(0)], then [O(j), S(j+1)]) is enqueued under the issue
      // lock once all its operands are ready, so the two streams' blocks reach
      // the tensor core whole and in turn: one stream's S completes a block
      // ahead of the other's and the two softmax groups run staggered instead
      // of contending for the same units.
      bool ok = !aborted && c.live;
      if (ok) ok = W.wait(&B.q_full[s][0], 0) && W.wait(&B.k_full[s], 0) && W.acquire(&sh.issue_lock);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tS, qdesc0 + (uint64_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4),
                      kdesc + (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4), idesc_s, k > 0 ? 1u : 0u);
        mma_commit(&B.k_empty[s]);
        mma_commit(&B.s_full[s]);
        atomicExch(&sh.issue_lock, 0);
        issued_any = true;
      } else if (c.live) {
        aborted = true;
      }
      while (!aborted && c.live) {
        // O of step j (P in TMEM, V in smem), then S of step j + 1.
        const bool first = (c.t == 0), last = (c.t == c.ntiles - 1);
        const int is = c.is;
        Cursor nx = c;
        cursor_next(p, nx);
        const int qb = nx.is & 1;
        if (!W.wait(&B.v_full[s], j & 1) || !W.wait(&B.p_full[s], j & 1) ||
            (first && is >= 1 && !W.wait(&B.o_empty[s], (is - 1) & 1)) ||
            (nx.live && nx.t == 0 && !W.wait(&B.q_full[s][qb], (nx.is >> 1) & 1)) ||
            (nx.live && !W.wait(&B.k_full[s], (j + 1) & 1)) || !W.acquire(&sh.issue_lock)) {
          aborted = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 8 steps of 16 keys; P step k = 8 TMEM columns
          mma_bf16_ts(tO, tS + 8u * k, vdesc + (uint64_t)((k * 2048) >> 4), idesc_o, (first && k == 0) ? 0u : 1u);
        mma_commit(&B.v_empty[s]);
        if (last) mma_commit(&B.o_full[s]);
        if (nx.live) {
          const uint64_t qd = qdesc0 + (uint64_t)((qb * L::Q_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)  // steps of 16 along D
            mma_bf16_ss(tS, qd + (uint64_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4),
                        kdesc + (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4), idesc_s, k > 0 ? 1u : 0u);
          mma_commit(&B.k_empty[s]);
          mma_commit(&B.s_full[s]);
        }
        atomicExch(&sh.issue_lock, 0);
        ++j;
        c = nx;
      }
      // Drain: every MMA issued by this thread completes before TMEM is released.
      if (issued_any) {
        mma_commit(&B.drain[s]);
        W.drain_wait(&B.drain[s], 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax (stream s)
    regs_inc<152>();
    const int s = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tSP = tmem + kColSP + 128u * s + lane_base;
    const uint32_t tO = tmem + kColO + 128u * s + lane_base;
    const float scale = p.scale_log2;
    int tc = 0;  // steps processed by this stream
    Cursor c;
    cursor_init(p, c, s);
    while (c.live) {
      const int n = c.n, ntiles = c.ntiles, is = c.is;
      float m0 = -INFINITY, m1 = -INFINITY;  // reference max (scaled) of rows a and a+8
      float l0 = 0.f, l1 = 0.f;              // this thread's share of the row sums
      for (int t = 0; t < ntiles; ++t, ++tc) {
        W.wait(&B.s_full[s], tc & 1);
        tc_fence_after();
        uint32_t r[64];
        ld_16x256b_x16(tSP, r);
        tmem_wait_ld();
        const bool tail = (2 * t + 1 >= n);
        if (tail) {
          // Odd tail: keys 64..127 (the repeated cube) do not take part.
#pragma unroll
          for (int e = 32; e < 64; ++e) r[e] = __float_as_uint(-INFINITY);
        }
        // Optimistic pass with the current reference max. A thread's partial
        // row sum exceeds 2^8 whenever one of its scores exceeds the reference
        // by more than 2^8 (and when the reference is still -inf), so only then
        // is the exact row max needed.
        uint32_t pk[32];
        float s0, s1;
        if (tail) exp_pack<false>(r, scale, m0, m1, pk, s0, s1);
        else exp_pack<true>(r, scale, m0, m1, pk, s0, s1);
        if (__any_sync(0xffffffffu, !(s0 <= 256.f) || !(s1 <= 256.f))) {
          float x0, x1;
          row_max(r, x0, x1);
          x0 *= scale;
          x1 *= scale;
          // Lazy reference update per row.
          float a0 = 1.f, a1 = 1.f;
          const bool u0 = x0 > m0 + 8.0f, u1 = x1 > m1 + 8.0f;
          if (u0) { a0 = fast_exp2(m0 - x0); m0 = x0; l0 *= a0; }
          if (u1) { a1 = fast_exp2(m1 - x1); m1 = x1; l1 *= a1; }
          if (__any_sync(0xffffffffu, u0 || u1)) {
            if (t > 0) {
              // O holds steps < t of this item (their MMAs completed before
              // this step's S): rescale the rows in place, 64 columns at a time.
#pragma unroll
              for (int h = 0; h < D / 64; ++h) {
                uint32_t o[32];
                ld_16x256b_x8(tO + 64u * h, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  o[4 * e] = __float_as_uint(__uint_as_float(o[4 * e]) * a0);
                  o[4 * e + 1] = __float_as_uint(__uint_as_float(o[4 * e + 1]) * a0);
                  o[4 * e + 2] = __float_as_uint(__uint_as_float(o[4 * e + 2]) * a1);
                  o[4 * e + 3] = __float_as_uint(__uint_as_float(o[4 * e + 3]) * a1);
                }
                st_16x256b_x8(tO + 64u * h, o);
              }
              tmem_wait_st();
            }
            if (tail) exp_pack<false>(r, scale, m0, m1, pk, s0, s1);
            else exp_pack<true>(r, scale, m0, m1, pk, s0, s1);
          }
        }
        l0 += s0;
        l1 += s1;
        st_16x128b_x16(tSP, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[s]);
      }
      // Row sums of the item -> 1/l for the epilogue.
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if ((lane & 3) == 0) {
        const int row = quarter * 16 + (lane >> 2);
        sh.inv_l[s][is & 1][row] = 1.0f / l0;
        sh.inv_l[s][is & 1][row + 8] = 1.0f / l1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.l_full[s][is & 1]);
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
    int qloads[2][2] = {{0, 0}, {0, 0}};
    // Q of item `is` of stream s -> smem buffer [s][is & 1] (TMA, one thread).
    auto load_q = [&](int s, int is) {
      const int item = blockIdx.x + (s + 2 * is) * gridDim.x;
      if (item >= p.n_items) return;
      const int b = is & 1;
      ++qloads[s][b];
      if (est == 0) {
        uint8_t* dst = tiles + L::OFF_Q + (2 * s + b) * L::Q_BYTES;
        mbar_arrive_expect_tx(&B.q_full[s][b], L::Q_BYTES);
#pragma unroll
        for (int h = 0; h < L::NH; ++h) tma_load_2d(dst + h * 8192, &p.tm_q, &B.q_full[s][b], 64 * h, item * 64);
      }
    };
    for (int s = 0; s < 2; ++s) {
      load_q(s, 0);
      load_q(s, 1);
    }
    // Items are finished in whatever order the two streams complete them (a
    // fixed order would let a long item of one stream hold back the other
    // stream's O buffer). Thread 0 of the group picks the stream; the group
    // follows through shared memory.
    int next_is[2] = {0, 0};
    while (true) {
      const bool live0 = blockIdx.x + (2 * next_is[0]) * gridDim.x < p.n_items;
      const bool live1 = blockIdx.x + (1 + 2 * next_is[1]) * gridDim.x < p.n_items;
      if (!live0 && !live1) break;
      if (est == 0) {
        int pick = live0 ? 0 : 1;
        if (live0 && live1) {
          const uint64_t t0 = globaltimer_ns();
          pick = -1;
          while (pick < 0) {
            if (mbar_try_wait(&B.o_full[0], next_is[0] & 1)) pick = 0;
            else if (mbar_try_wait(&B.o_full[1], next_is[1] & 1)) pick = 1;
            else if (*(volatile int*)&sh.abort_flag || globaltimer_ns() - t0 > p.wait_ns) pick = 0;
          }
        }
        sh.epi_pick = pick;
      }
      epi_sync();
      const int s = sh.epi_pick;
      const int is = next_is[s]++;
      const int item = blockIdx.x + (s + 2 * is) * gridDim.x;
      const int bh = item / C, ci = item - bh * C;
      // raster token of the cube's first row; row q adds ((q>>4)*H + (q>>2&3))*W + (q&3)
      const int ct = ci / (Hc * Wc), ch = (ci / Wc) % Hc, cw = ci % Wc;
      const int tok_base = ((4 * ct) * p.H + 4 * ch) * p.W + 4 * cw;
      auto tok_of = [&](int q) { return tok_base + ((q >> 4) * p.H + ((q >> 2) & 3)) * p.W + (q & 3); };
      const int tok0 = tok_of(ra), tok1 = tok_of(ra + 8);
      const float gc0 = p.gate_c[(size_t)bh * p.N + tok0], gf0 = p.gate_f[(size_t)bh * p.N + tok0];
      const float gc1 = p.gate_c[(size_t)bh * p.N + tok1], gf1 = p.gate_f[(size_t)bh * p.N + tok1];
      const float* ocrow = p.oc + ((size_t)bh * C + ci) * D;
      W.wait(&B.l_full[s][is & 1], (is >> 1) & 1);
      const float il0 = sh.inv_l[s][is & 1][ra], il1 = sh.inv_l[s][is & 1][ra + 8];
      W.wait(&B.o_full[s], is & 1);
      tc_fence_after();
      float o[2 * D / 4];
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t r[32];
        ld_16x256b_x8(tmem + kColO + 128u * s + 64u * h + lane_base, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[32 * h + j] = __uint_as_float(r[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.o_empty[s]);
      // All S steps of this item completed: its Q buffer takes the stream's item after next.
      load_q(s, is + 2);
      // o[4j..4j+3] = (row ra: d, d+1; row ra+8: d, d+1), d = 8j + 2 tq
      if (p.out_fine) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const int d = 8 * j + 2 * tq;
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok0) * D + d) =
              make_float2(o[4 * j] * il0, o[4 * j + 1] * il0);
          *reinterpret_cast<float2*>(p.out_fine + ((size_t)bh * p.N + tok1) * D + d) =
              make_float2(o[4 * j + 2] * il1, o[4 * j + 3] * il1);
        }
      }
      if (p.out) {
        const float f0 = gf0 * il0, f1 = gf1 * il1;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const int d = 8 * j + 2 * tq;
          const float2 oc = *reinterpret_cast<const float2*>(ocrow + d);
          const __nv_bfloat162 h0 =
              __floats2bfloat162_rn(fmaf(gc0, oc.x, f0 * o[4 * j]), fmaf(gc0, oc.y, f0 * o[4 * j + 1]));
          const __nv_bfloat162 h1 =
              __floats2bfloat162_rn(fmaf(gc1, oc.x, f1 * o[4 * j + 2]), fmaf(gc1, oc.y, f1 * o[4 * j + 3]));
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
          *reinterpret_cast<uint4*>(p.out + ((size_t)bh * p.N + tok_of(q)) * D + off * 8) = v;
        }
      }
      epi_sync();  // staging reads and the stream pick are done before the next item
    }
    // Drain: the last Q copy of each buffer has landed (it has, unless the run aborted).
    if (est == 0)
      for (int s2 = 0; s2 < 2; ++s2)
        for (int b = 0; b < 2; ++b)
          if (qloads[s2][b] > 0) W.drain_wait(&B.q_full[s2][b], (qloads[s2][b] - 1) & 1);
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
