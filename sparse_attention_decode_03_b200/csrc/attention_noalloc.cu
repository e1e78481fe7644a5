// qsa_sparse_attention_noalloc: qsa_sparse_decode followed by qsa_combine, with
// the split partials kept in a device array that this file reserves, so the
// caller passes only inputs and outputs and allocates nothing.
//
// Who needs this: a caller that cannot call cudaMalloc.  Examples are a serving
// engine that gives nearly all device memory to its KV-cache pool at start-up,
// leaving no room for per-step buffers; a plug-in whose host application owns
// every device allocation; and a latency-critical loop where cudaMalloc's
// implicit device synchronisation is not allowed.
//
// The array: a file-scope __device__ array of QSA_NOALLOC_SCRATCH_BYTES.  The
// module holds it on every GPU that loads the library until the process exits.
// Host code cannot pass the array's name to a kernel: on the host that name is
// only a stand-in symbol, not a device address.  So the first call on each
// device, with that device current, asks the runtime for the array's device
// address (cudaGetSymbolAddress) and caches it per device.  Make that first
// call before any stream capture.
//
// Every call on a device shares the one array and leaves its contents behind.
// The decode writes every partial slot that the combine then reads, so nothing
// has to be cleared between calls.  Calls whose kernels can overlap on the GPU
// (unordered streams, several host threads) race on the array: order them on
// one stream.
#include "qsa_common.cuh"

#include <mutex>

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_partials[QSA_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_partials on the current device (looked up once per device).
int partials_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return QSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_partials);
    if (e != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return QSA_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return QSA_OK;
}

}  // namespace

int32_t qsa_splits_bound(int32_t k, int32_t chunk);

extern "C" int qsa_sparse_attention_noalloc(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq,
                                            const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel,
                                            const int32_t* count, int32_t k, float scale, int32_t chunk_units,
                                            void* out, float* lse, int32_t* dev_status, void* stream) {
  if (nq < 0 || hq < 1 || k < 0 || k > QSA_MAX_TOPK || chunk_units < 1) return QSA_ERR_INVALID_ARG;
  if (!out || !lse || (reinterpret_cast<uintptr_t>(out) & 7u)) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  const int32_t splits = qsa_splits_bound(k, chunk_units);
  // part_o [nq][splits][hq][256] fp32, then part_lse [nq][splits][hq] fp32
  const uint64_t rows = (uint64_t)nq * (uint64_t)splits * (uint64_t)hq;
  const uint64_t o_bytes = rows * QSA_HEAD_DIM * sizeof(float);
  const uint64_t need = o_bytes + rows * sizeof(float);
  if (need > (uint64_t)QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_UNSUPPORTED;
  void* base = nullptr;
  const int rc = partials_address(&base);
  if (rc != QSA_OK) return rc;
  float* part_o = static_cast<float*>(base);
  float* part_lse = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + o_bytes);
  const int rd = qsa_sparse_decode(cache, q, nq, hq, q_seq, q_pos, sel, count, k, scale, chunk_units, splits,
                                   part_o, part_lse, dev_status, stream);
  if (rd != QSA_OK) return rd;
  return qsa_combine(part_o, part_lse, nq, splits, hq, out, lse, stream);
}
