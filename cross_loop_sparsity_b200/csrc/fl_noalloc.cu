// fl_noalloc.cu -- the skinny (decode-shaped) GEMM for callers that cannot
// allocate device memory.
//
// Some callers may not call cudaMalloc at all: code that runs inside another
// framework's memory pool which already owns all device memory, latency-
// critical paths that cannot afford cudaMalloc's implicit device
// synchronisation, or plugin hosts that forbid allocation.  The split-K GEMM
// otherwise needs caller-provided scratch for its partial tiles and tickets.
// This entry point keeps that scratch in a fixed array compiled into the
// library instead: every GPU that loads the library holds it until the
// process exits, and no call allocates anything.
#include <cstring>
#include <mutex>
#include <string>

#include "flashloop.h"
#include "fl_internal.h"

namespace {

// Split-K partial tiles (floats) followed by the per-tile tickets.
constexpr size_t kPartialBytes = FL_NOALLOC_SCRATCH_BYTES;
constexpr size_t kTicketBytes = 4096 * sizeof(int);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kPartialBytes + kTicketBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};  // device address of g_noalloc_scratch, per device

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

// Failures leave their reason where flashloop_last_cuda_error(NULL) reports it.
fl_status fail(fl_status st, const std::string& why) {
  fl::set_last_error(why);
  return st;
}

}  // namespace

extern "C" {

fl_status fl_gemm_skinny_noalloc(const uint16_t* A, const uint16_t* B, float* D, int m, int n, int k,
                                 fl_stream_t stream) {
  if (!A || !B || !D || m < 1 || m > 64 || n < 1 || k < 8 || k % 8)
    return fail(FL_ERR_INVALID_ARG, "A, B, D must be non-NULL; 1 <= m <= 64; k >= 8 and a multiple of 8");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(D)) & 15)
    return fail(FL_ERR_INVALID_ARG, "A, B and D must be 16-byte aligned");
  // the same tile width and split rule as fl_test_gemm, so both give the same product bit for bit
  const int bn = fl::swap_bn(m);
  const int tiles = ceil_div(n, 128);
  const int k_chunks = ceil_div(k, 64);
  const int splits = fl::split_factor(tiles, k_chunks);
  const size_t need = fl::gemm_partial_floats(bn, 0, tiles, splits) * sizeof(float);
  if (need > kPartialBytes || static_cast<size_t>(tiles) * sizeof(int) > kTicketBytes)
    return fail(FL_ERR_CAPACITY, "this shape needs " + std::to_string(need) + " bytes of split-K scratch; the "
                "built-in array holds " + std::to_string(kPartialBytes) + " (use fl_test_gemm with caller scratch)");
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return fail(FL_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = fl::gemm_init_attrs();
  if (e != cudaSuccess) return fail(FL_ERR_CUDA, cudaGetErrorString(e));
  CUtensorMap ta, tb;
  if (!fl::encode_tmap_bf16(&ta, B, k, n, 0, 128) || !fl::encode_tmap_bf16(&tb, A, k, m, 0, bn))
    return fail(FL_ERR_INVALID_ARG, "tensor map encoding failed");
  int* tickets = reinterpret_cast<int*>(static_cast<unsigned char*>(base) + kPartialBytes);
  if (splits > 1) {
    // tickets must start at zero; a previous call normally leaves them zero,
    // but they are cleared here so an interrupted call cannot poison the next
    e = cudaMemsetAsync(tickets, 0, static_cast<size_t>(tiles) * sizeof(int), s);
    if (e != cudaSuccess) return fail(FL_ERR_CUDA, cudaGetErrorString(e));
  }
  fl::GemmLaunch g{};
  fl::GemmArgs& a = g.args;
  a.k_chunks = k_chunks;
  a.splits = splits;
  a.swap = 1;
  a.epi = fl::kEpiStore;
  a.n_feat = n;
  a.n_tok = m;
  a.out = D;
  a.ldo = n;
  a.partial = static_cast<float*>(base);
  a.counters = tickets;
  g.a0 = &ta;
  g.b0 = &tb;
  g.bn = bn;
  g.grid = dim3(tiles, 1, splits);
  e = fl::launch_gemm(g, s);
  if (e != cudaSuccess) return fail(FL_ERR_CUDA, cudaGetErrorString(e));
  return FL_OK;
}

}  // extern "C"
