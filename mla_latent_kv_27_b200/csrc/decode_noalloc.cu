// mla_decode_attention_noalloc: the split-KV decode with its partials kept in a static
// device buffer of this library instead of a caller workspace, for callers that cannot
// allocate device memory.  The kernels are those of mla_decode_attention.
#include <atomic>

#include "mla_internal.cuh"

namespace mla {

// The scratch: one per device that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

// In host code g_noalloc_scratch names a host-side stand-in, not the device buffer; the
// device address is looked up once per device, with that device current.
static void* noalloc_scratch(mla_status* status) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = MLA_ERR_CUDA;
    return nullptr;
  }
  static std::atomic<void*> addr[64];
  void* p = addr[dev].load(std::memory_order_acquire);
  if (!p) {
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      *status = MLA_ERR_CUDA;
      return nullptr;
    }
    addr[dev].store(p, std::memory_order_release);
  }
  *status = MLA_OK;
  return p;
}

}  // namespace mla

extern "C" mla_status mla_decode_attention_noalloc(const mla_dims* dims, const void* q_packed,
                                                   const mla_cache* cache, const int32_t* seq_lens,
                                                   int32_t batch, int32_t s_q, int32_t causal,
                                                   int32_t n_split, void* o_lat, float* lse,
                                                   void* stream) {
  if (!cache) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_decode_workspace_size(dims, batch, s_q, n_split, cache->max_pages_per_seq);
  if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_UNSUPPORTED;
  mla_status st = MLA_OK;
  void* scratch = need > 0 ? mla::noalloc_scratch(&st) : nullptr;
  if (st != MLA_OK) return st;
  return mla_decode_attention(dims, q_packed, cache, seq_lens, batch, s_q, causal, n_split, scratch,
                              need > 0 ? MLA_NOALLOC_SCRATCH_BYTES : 0, o_lat, lse, stream);
}
