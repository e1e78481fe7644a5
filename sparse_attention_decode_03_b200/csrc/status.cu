// Status strings, ABI version and the host-only decode planner.
#include "qsa_common.cuh"

extern "C" const char* qsa_status_string(int status) {
  switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    default: return "QSA_ERR_UNKNOWN";
  }
}

extern "C" int qsa_abi_version(void) { return QSA_ABI_VERSION; }

// Most chunks of `chunk` slots that a run of n = k+1 consecutive slots can touch.
static int32_t splits_bound(int32_t k, int32_t chunk) {
  const int64_t n = (int64_t)k + 1;
  return (int32_t)((n + chunk - 2) / chunk + 1);
}

extern "C" int qsa_decode_plan(int32_t nq, int32_t hkv, int32_t k, int32_t target_ctas, int32_t* chunk_units,
                               int32_t* max_splits) {
  if (!chunk_units || !max_splits || nq < 0 || hkv < 1 || k < 0 || k > QSA_MAX_TOPK || target_ctas < 1)
    return QSA_ERR_INVALID_ARG;
  const int64_t slots = (int64_t)nq * hkv * ((int64_t)k + 1);
  // Floor of 16 slots (64 KiB of K+V per KV head) keeps the per-split partial
  // (fp32 o and lse) small next to the bytes it summarises.
  int64_t chunk = (slots + target_ctas - 1) / target_ctas;
  if (chunk < 16) chunk = 16;
  if (chunk > (int64_t)1 << 30) chunk = (int64_t)1 << 30;
  *chunk_units = (int32_t)chunk;
  *max_splits = splits_bound(k, (int32_t)chunk);
  return QSA_OK;
}

// exported for the other translation units
int32_t qsa_splits_bound(int32_t k, int32_t chunk) { return splits_bound(k, chunk); }
