// Work order of the persistent fine-attention kernels when items differ in
// length.
//
// "Improving Video Sparse Attention with Fine-grained Router and Sparse
// Rebasing", "Abstract (arXiv)": each query may attend to a variable number
// of key-value blocks, so the items of the fine stage (one query cube and its
// selected KV cubes) have different lengths; so have the items of the dK/dV
// backward kernel (one KV cube and the query cubes that selected it) even
// with a fixed top-K. The persistent kernels give CTA c the positions
//   is * G + c            (is even)
//   is * G + G - 1 - c    (is odd)        G = grid size,
// of an order array, which lists each head's items by descending length
// (ties by ascending id), head after head. Longest first with a serpentine
// hand-out balances the CTAs' total work (each pair of rounds gives every CTA
// one long and one short item), and keeping the heads in sequence keeps one
// or two heads' K/V resident in L2 as the unordered walk does.
//
// One warp per (batch, head): a histogram of the lengths in shared memory, an
// exclusive scan from the longest length down, then a stable scatter of the
// item ids (lanes with equal lengths are ranked by lane order with
// __match_any_sync, and the ids are visited in ascending order).
#include "vsa_common.cuh"

namespace vsa {

namespace {

__global__ void __launch_bounds__(32) schedule_kernel(const int32_t* __restrict__ len, int32_t* __restrict__ order,
                                                      int C, int maxlen) {
  extern __shared__ int bins[];  // maxlen + 1 counters
  const int bh = blockIdx.x, lane = threadIdx.x;
  const int32_t* l = len + (size_t)bh * C;
  for (int i = lane; i <= maxlen; i += 32) bins[i] = 0;
  __syncwarp();
  for (int i = lane; i < C; i += 32) {
    int v = l[i];
    v = v < 0 ? 0 : (v > maxlen ? maxlen : v);
    atomicAdd(&bins[v], 1);
  }
  __syncwarp();
  // exclusive scan from the longest length down: bins[v] = first position of length v
  if (lane == 0) {
    int run = 0;
    for (int v = maxlen; v >= 0; --v) {
      const int c = bins[v];
      bins[v] = run;
      run += c;
    }
  }
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = 0; i0 < C; i0 += 32) {
    const int i = i0 + lane;
    const bool have = i < C;
    int v = have ? l[i] : -1;
    v = !have ? -1 : (v < 0 ? 0 : (v > maxlen ? maxlen : v));
    const unsigned active = __ballot_sync(0xffffffffu, have);
    const unsigned peers = __match_any_sync(0xffffffffu, v) & active;
    if (have) {
      const int rank = __popc(peers & lt);
      order[(size_t)bh * C + bins[v] + rank] = bh * C + i;
    }
    __syncwarp();
    // the lowest lane of each group of equal lengths advances the bin
    if (have && (peers & lt) == 0) bins[v] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_schedule(const int32_t* len, int32_t* order, int BH, int C, int maxlen, cudaStream_t st) {
  schedule_kernel<<<BH, 32, (size_t)(maxlen + 1) * sizeof(int), st>>>(len, order, C, maxlen);
  return cudaGetLastError();
}

}  // namespace vsa
