// rmt_memory_write_noalloc: the memory write of rmt_memory_write with no device allocation.
//
// Some callers cannot let a library call cudaMalloc: a serving engine or caching allocator
// that has already claimed the device's memory for its own pool (a cudaMalloc there can
// fail, and it synchronizes the whole device, stalling the caller's other streams). This
// entry point keeps its scratch -- the cell table and the split-K partial sums of the
// key/value projection -- in a fixed array in the library's own device memory instead.
#include <atomic>
#include <string>

#include "common.cuh"
#include "launch.h"
#include "rmt.h"

namespace {

using rmt::Cell;

// Scratch for rmt_memory_write_noalloc: the cell table, then the partial sums. With CUDA's
// lazy module loading (the default), a device gets these 8 MiB when this file's module is
// first loaded there -- at the first rmt_memory_write_noalloc call on that device -- and
// holds them until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr size_t kNoAllocCellBytes = 256 << 10;  // room for 8192 cells
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device (host code cannot use the
// symbol itself: on the host it names a stand-in, not device memory). Host threads may race
// on the first lookup; each stores the same address. The cached address belongs to the
// device's context of the time: it does not survive a cudaDeviceReset of that device.
std::atomic<void*> g_noalloc_addr[64] = {};

__global__ void fill_cells_kernel(Cell* cells, int G) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g < G) cells[g] = rmt::identity_cell(g);
}

}  // namespace

namespace rmt {
void set_last_error(const std::string& msg);
}

extern "C" rmt_status rmt_memory_write_noalloc(const float* y, const void* w_mkv, float* A, float* z, int32_t G,
                                               int32_t n, int32_t d, int32_t dk, int32_t dv, float eps,
                                               rmt_dtype dtype, void* stream) {
  auto fail = [](rmt_status st, const char* msg) {
    rmt::set_last_error(msg);
    return st;
  };
  if (!y || !w_mkv || !A || !z) return fail(RMT_EINVAL, "null pointer");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(z)) & 15u)
    return fail(RMT_EINVAL, "A and z must be 16-byte aligned");
  if (G <= 0 || n <= 0 || n > 64 || d <= 0 || dk <= 0 || dv <= 0 || dk % 32 || dv % 32 || dk > 128 || dv > 128 ||
      n * (dk + dv) > 4096)
    return fail(RMT_EINVAL, "bad sizes");
  if (dtype != RMT_F32 && dtype != RMT_BF16) return fail(RMT_EINVAL, "bad dtype");
  // the projection writes ceil(d/128) partial sums per cell, or their whole sum when the launch is
  // large (mem_kv_written_splits)
  const size_t nsplit = static_cast<size_t>(rmt::mem_kv_written_splits(G, n, d, dtype == RMT_BF16));
  const size_t part_bytes = size_t(G) * nsplit * n * (dk + dv) * sizeof(float);
  if (size_t(G) * sizeof(Cell) > kNoAllocCellBytes || part_bytes > kNoAllocScratchBytes - kNoAllocCellBytes)
    return fail(RMT_EINVAL,
                "rmt_memory_write_noalloc: G*splits*n*(dk+dv)*4 bytes of partial sums exceed the fixed "
                "8 MiB - 256 KiB scratch (or G > 8192); use rmt_memory_write");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(RMT_ECUDA, "cudaGetDevice failed");
  void* addr = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (!addr) {
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess || !addr)
      return fail(RMT_ECUDA, "rmt_memory_write_noalloc: cudaGetSymbolAddress of the scratch array failed");
    g_noalloc_addr[dev].store(addr, std::memory_order_release);
  }
  unsigned char* base = static_cast<unsigned char*>(addr);
  Cell* cells = reinterpret_cast<Cell*>(base);
  float* part = reinterpret_cast<float*>(base + kNoAllocCellBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The cell table is rewritten on every call; the partial sums need no clearing because
  // the projection kernel writes every element the update kernel reads.
  fill_cells_kernel<<<(G + 255) / 256, 256, 0, st>>>(cells, G);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    rmt::MemKvArgs ka{y, n, d, n, rmt::kByLayer, w_mkv, part, dk + dv, G, cells, G};
    e = rmt::launch_mem_kv(ka, dtype == RMT_BF16, st);
  }
  if (e == cudaSuccess) {
    rmt::MemUpdateArgs ua{part, int(nsplit), nullptr, nullptr, A, z, n, dk, dv, eps, G, cells, rmt::kByLayer,
                          rmt::kByLayer, G, nullptr, 0, 0};
    e = rmt::launch_mem_update(ua, st);
  }
  if (e != cudaSuccess) return fail(RMT_ECUDA, cudaGetErrorString(e));
  return RMT_OK;
}
