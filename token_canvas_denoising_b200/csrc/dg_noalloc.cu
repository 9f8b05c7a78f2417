// dg_lmhead_entropy_noalloc: the fused LM head + entropy/argmax without any
// device allocation. Some callers cannot allocate device memory at the point
// where they need this operation: applications whose device memory is fully
// reserved up front by their own allocator, where a driver allocation in the
// middle of a step fails or fragments what is left; and hosts that give a
// plug-in only the buffers they pass it and forbid it to allocate (or to pay
// the device-wide synchronisation an allocation can cost). For them the
// per-CTA partial results that dg_lmhead_entropy keeps in a temporary buffer
// live in a fixed, library-owned device array instead.
#include "dg_internal.cuh"
#include "dg_ops.h"

namespace {

// Scratch for the per-(row, vocab partition) partial records. It is a
// file-scope device array: every GPU that loads the library holds it (2 MiB)
// until the process exits, and every call on that GPU shares it.
constexpr size_t kScratchRecords = 65536;
static __device__ __align__(256) dg::LmRec g_lm_scratch[kScratchRecords];
// Device error word of this entry point's kernels (a bounded wait that gave
// up, a NaN entropy), read and cleared by dg_ops_check.
static __device__ int g_noalloc_err;

// In host code the names above are host-side stand-ins, not device
// addresses: the addresses are looked up per device and context (the first
// call on each device does it) and passed to the kernels.
dg::SymbolAddressCache g_scratch_addr, g_err_addr;

}  // namespace

namespace dg {
dg_status noalloc_error_word(int** out) {
  void* p = nullptr;
  const dg_status st = g_err_addr.get(g_noalloc_err, &p);
  *out = static_cast<int*>(p);
  return st;
}
}  // namespace dg

extern "C" {

size_t dg_lmhead_entropy_noalloc_max_records(void) { return kScratchRecords; }

dg_status dg_lmhead_entropy_noalloc(int32_t dtype, const void* hs, const void* lm_head, const float* inv_temp,
                                    int32_t M, int32_t d, int32_t V, float* ent, int32_t* argmax, void* stream) {
  if (!(dtype == DG_F32 || dtype == DG_BF16) || !hs || !lm_head || !ent || !argmax || M < 1 || d < 1 || V < 2) {
    dg::set_last_error("invalid argument: dtype, NULL buffer or sizes");
    return DG_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(hs) & 15u) || (reinterpret_cast<uintptr_t>(lm_head) & 15u)) {
    dg::set_last_error("invalid argument: hs / lm_head must be 16-byte aligned");
    return DG_ERR_INVALID_ARG;
  }
  if (d % 8 != 0 || (dtype == DG_BF16 && (d % 64 != 0 || V % 256 != 0))) {
    dg::set_last_error("unsupported: d % 8 (bf16: d % 64 and V % 256)");
    return DG_ERR_UNSUPPORTED;
  }
  dg::Exec ex;
  ex.stream = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&ex.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    dg::set_last_error("no usable CUDA device");
    return DG_ERR_CUDA;
  }
  dg::LmPartials part;
  part.P = dtype == DG_BF16 ? dg::lmhead_tc_partitions(M, V, ex.sm_count) : std::max(1, std::min(128, V / 1024));
  if ((size_t)M * (size_t)part.P > kScratchRecords) {
    dg::set_last_error("unsupported: M * vocab partitions = " + std::to_string((size_t)M * part.P) +
                       " exceeds the fixed scratch of " + std::to_string(kScratchRecords) + " records");
    return DG_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  dg_status st = g_scratch_addr.get(g_lm_scratch, &scratch);
  if (st == DG_OK) st = dg::noalloc_error_word(&ex.err);
  if (st != DG_OK) return st;
  // every record the merge reads is written by this call's LM-head kernel, so
  // nothing left in the array by an earlier call is read
  part.rec = static_cast<dg::LmRec*>(scratch);
  if (dtype == DG_BF16) {
    CUtensorMap a, b;
    if (!dg::lmhead_tc_prepare(hs, lm_head, M, d, V, &a, &b)) return DG_ERR_CUDA;
    dg::launch_lmhead_tc(ex, a, b, part, inv_temp, M, d, V);
  } else {
    dg::launch_lmhead_simple(ex, dtype, hs, lm_head, inv_temp, part, M, d, V);
  }
  dg::launch_merge_select(ex, part, ent, argmax, nullptr, nullptr, nullptr, 1, M, V);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    dg::set_last_error(std::string("launch: ") + cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

}  // extern "C"
