// Measurement kernel: L2 -> SM read bandwidth of bulk (TMA-engine) copies.
//
// The fine-attention kernel streams every selected K/V tile from L2 into
// shared memory with TMA, 64 FLOP of tensor work per byte, so the rate at
// which L2 can feed the SMs bounds it next to the tensor pipe. This kernel
// reads a buffer that is resident in L2 the same way: each CTA has one thread
// that keeps a ring of 16 KB untiled bulk copies (global -> this CTA's shared
// memory, completion on an mbarrier) in flight over its share of the buffer's
// chunks, for a given number of passes. Nothing is computed on the data.
// Every wait is bounded; a wait that gives up sets *status and the CTA
// returns after waiting (bounded) for the copies it issued.
#include "sm100_ptx.cuh"
#include "vsa_common.cuh"

namespace vsa {

namespace {

constexpr int kChunk = 16384;
constexpr int kRing = 6;

__global__ void __launch_bounds__(32, 1)
    l2_read_kernel(const uint8_t* buf, long long nchunks, int passes, int* status, unsigned long long wait_ns) {
  using namespace ptx;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kRing];
  if (threadIdx.x != 0) return;
  for (int i = 0; i < kRing; ++i) mbar_init(&full[i], 1);
  fence_mbar_init();
  const long long per_pass = (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const long long total = blockIdx.x < nchunks ? per_pass * passes : 0;
  long long issued = 0;
  bool ok = true;
  for (long long i = 0; i < total; ++i) {
    const int slot = (int)(i % kRing);
    if (i >= kRing && !mbar_wait(&full[slot], (uint32_t)(((i / kRing) - 1) & 1), wait_ns)) {
      ok = false;
      break;
    }
    const long long c = blockIdx.x + (i % per_pass) * gridDim.x;
    const uint8_t* src = buf + c * kChunk;
    mbar_arrive_expect_tx(&full[slot], kChunk);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_raw + slot * kChunk)),
        "l"(src), "r"(kChunk), "r"(smem_u32(&full[slot]))
        : "memory");
    ++issued;
  }
  // Wait for the last phase armed in each slot (phases complete in order).
  for (int slot = 0; slot < kRing && slot < issued; ++slot) {
    const long long uses = (issued - 1 - slot) / kRing + 1;
    if (!mbar_wait(&full[slot], (uint32_t)((uses - 1) & 1), wait_ns)) ok = false;
  }
  if (!ok) atomicOr(status, 1);
}

}  // namespace

cudaError_t launch_l2_read(const void* buf, size_t bytes, int passes, int* status, int grid, cudaStream_t st) {
  const int smem = kRing * kChunk;
  cudaError_t e = cudaFuncSetAttribute(l2_read_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  l2_read_kernel<<<grid, 32, smem, st>>>(static_cast<const uint8_t*>(buf), (long long)(bytes / kChunk), passes,
                                         status, 1000000000ull);
  return cudaGetLastError();
}

}  // namespace vsa
