// C ABI of libmla: argument validation, dispatch to the kernels, workspace sizing and the
// per-device error word.  Declarations and their contracts are in include/mla.h.
#include <atomic>
#include <cstdio>
#include <cstring>

#include <cstdlib>

#include "mla_internal.cuh"
#include "decode_tc.cuh"

namespace mla {

static std::atomic<unsigned long long> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// Per-device error word (each device that loads the module gets its own copy).
__device__ int g_error_word = 0;

// The word's device address, looked up once per device (with that device current) and cached;
// threads that race on a device's first call store the same address.  The cache assumes the
// device's primary context lives as long as the process (no cudaDeviceReset in between).
static int* error_word_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  static std::atomic<int*> ptrs[64];
  if (dev < 0 || dev >= 64) return nullptr;
  int* p = ptrs[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_error_word) != cudaSuccess || !a) return nullptr;
    p = static_cast<int*>(a);
    ptrs[dev].store(p, std::memory_order_release);
  }
  return p;
}

static bool dtype_ok(int t) { return t == MLA_F32 || t == MLA_BF16 || t == MLA_FP8_E4M3; }

static mla_status check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->d_model <= 0 || d->d_c <= 0 || d->d_rope <= 0 || d->d_nope <= 0 || d->d_v <= 0 ||
      d->n_heads <= 0 || d->page_size <= 0)
    return MLA_ERR_INVALID_ARG;
  if (d->d_rope % 2) return MLA_ERR_INVALID_ARG;
  if (!dtype_ok(d->act_dtype) || !dtype_ok(d->cache_dtype)) return MLA_ERR_INVALID_ARG;
  if (d->act_dtype == MLA_FP8_E4M3) return MLA_ERR_UNSUPPORTED;
  if (d->cache_dtype == MLA_F32 && d->act_dtype != MLA_F32) return MLA_ERR_UNSUPPORTED;
  if (d->act_dtype == MLA_F32 && d->cache_dtype != MLA_F32) return MLA_ERR_UNSUPPORTED;
  if (d->cache_dtype == MLA_FP8_E4M3 && d->d_c % 128) return MLA_ERR_UNSUPPORTED;
  if (!(d->scale == d->scale)) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

static mla_status check_cache(const mla_dims* d, const mla_cache* c) {
  if (!c || !c->rows || !c->block_table) return MLA_ERR_INVALID_ARG;
  if (c->max_pages_per_seq <= 0 || c->num_pages <= 0 || c->num_seqs <= 0) return MLA_ERR_INVALID_ARG;
  if (d->cache_dtype == MLA_FP8_E4M3 && (!c->scales || !c->rope)) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

static CacheView make_view(const mla_dims* d, const mla_cache* c) {
  CacheView v;
  v.rows = c->rows;
  v.scales = c->scales;
  v.rope = c->rope;
  v.block_table = c->block_table;
  v.max_pages = c->max_pages_per_seq;
  v.num_pages = c->num_pages;
  v.num_seqs = c->num_seqs;
  v.page_size = d->page_size;
  v.kind = d->cache_dtype;
  return v;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MLA_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

static mla_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  if (e == kUnsupported) return MLA_ERR_UNSUPPORTED;
  return MLA_ERR_CUDA;
}

// Decode split policy of the general kernel: enough CTAs for two waves on 148 SMs.
static int simt_auto_split(const mla_dims* d, int batch, int s_q, int max_pages) {
  int hpc = decode_simt_heads_per_cta(d->n_heads, s_q);
  long ctas = (long)batch * (d->n_heads / hpc);
  int n = (int)((2 * 148 + ctas - 1) / ctas);
  if (n < 1) n = 1;
  if (n > max_pages) n = max_pages;
  if (n > 64) n = 64;
  return n;
}

static int effective_split(const mla_dims* d, int batch, int s_q, int n_split, int max_pages) {
  if (n_split > 0) return n_split;
  return simt_auto_split(d, batch, s_q, max_pages);
}

// The two partitioned kernels: the small-head one (at most 16 heads, bf16) and the tcgen05 one.
// Both always run the length-balanced partition, whatever n_split says.
enum class DecodePath { General, SmallHead, TensorCore };
static DecodePath decode_path(const mla_dims* d) {
  if (sh_decode_supported(*d, d->cache_dtype)) return DecodePath::SmallHead;
  if (tc_decode_supported(*d, d->cache_dtype)) return DecodePath::TensorCore;
  return DecodePath::General;
}
static bool partitioned(const mla_dims* d) { return decode_path(d) != DecodePath::General; }

}  // namespace mla

using namespace mla;

extern "C" {

int32_t mla_version(void) { return 100; }

uint64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MLA_ERR_CUDA: return "CUDA runtime error";
    case MLA_ERR_DEVICE: return "device-side data error (bad page id, position or sequence)";
    case MLA_ERR_TIMEOUT: return "device-side bounded wait timed out";
  }
  return "unknown status";
}

mla_status mla_check_device_error(void* stream, int32_t* detail) {
  if (detail) *detail = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  int* p = error_word_ptr();
  if (!p) return MLA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (word == 0) return MLA_OK;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MLA_ERR_CUDA;
  if (detail) *detail = word;
  return (word >> 24) == ERR_TIMEOUT ? MLA_ERR_TIMEOUT : MLA_ERR_DEVICE;
}

mla_status mla_rope_table(int32_t d_rope, int32_t max_pos, float theta, float* cos_out,
                          float* sin_out, void* stream) {
  if (d_rope <= 0 || d_rope % 2 || max_pos <= 0 || !(theta > 0.f) || !cos_out || !sin_out)
    return MLA_ERR_INVALID_ARG;
  return cuda_status(launch_rope_table(d_rope, max_pos, theta, cos_out, sin_out,
                                       static_cast<cudaStream_t>(stream)));
}

size_t mla_append_workspace_size(const mla_dims* dims, int32_t n_tok) {
  if (check_dims(dims) != MLA_OK || n_tok < 0) return 0;
  return append_workspace_bytes(*dims, n_tok);
}

mla_status mla_append_cache(const mla_dims* dims, const void* h, int32_t n_tok,
                            const int32_t* seq_idx, const int32_t* pos, const void* w_dkv,
                            const void* w_kr, const float* rope_cos, const float* rope_sin,
                            int32_t rope_rows, const mla_cache* cache, void* workspace,
                            size_t workspace_bytes, void* stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if ((s = check_cache(dims, cache)) != MLA_OK) return s;
  if (!h || !seq_idx || !pos || !w_dkv || !w_kr || !rope_cos || !rope_sin || rope_rows <= 0)
    return MLA_ERR_INVALID_ARG;
  const size_t need = append_workspace_bytes(*dims, n_tok);
  if (workspace_bytes < need || (need > 0 && !workspace)) return MLA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (!err) return MLA_ERR_CUDA;
  return cuda_status(launch_append(*dims, h, n_tok, seq_idx, pos, w_dkv, w_kr, rope_cos, rope_sin,
                                   rope_rows, make_view(dims, cache), static_cast<float*>(workspace),
                                   err, static_cast<cudaStream_t>(stream)));
}

mla_status mla_absorb_query(const mla_dims* dims, const void* q_nope, const void* q_rope,
                            const int32_t* q_pos, int32_t n_tok, const void* w_uk,
                            const float* rope_cos, const float* rope_sin, int32_t rope_rows,
                            void* q_packed, void* stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!q_nope || !q_rope || !q_pos || !w_uk || !rope_cos || !rope_sin || rope_rows <= 0 || !q_packed)
    return MLA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (!err) return MLA_ERR_CUDA;
  return cuda_status(launch_absorb(*dims, q_nope, q_rope, q_pos, n_tok, w_uk, rope_cos, rope_sin,
                                   rope_rows, q_packed, err, static_cast<cudaStream_t>(stream)));
}

size_t mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t s_q,
                                 int32_t n_split, int32_t max_pages_per_seq) {
  if (check_dims(dims) != MLA_OK || batch < 0 || s_q <= 0 || n_split < 0 || max_pages_per_seq <= 0)
    return 0;
  if (decode_path(dims) == DecodePath::SmallHead) return sh_plan_workspace_bytes(*dims, batch, s_q);
  if (decode_path(dims) == DecodePath::TensorCore) return tc_plan_workspace_bytes(*dims, batch, s_q);
  int n = effective_split(dims, batch, s_q, n_split, max_pages_per_seq);
  if (n <= 1) return 0;
  size_t rows = (size_t)batch * n * s_q * dims->n_heads;
  return rows * dims->d_c * sizeof(float) + rows * sizeof(float);
}

mla_status mla_decode_attention(const mla_dims* dims, const void* q_packed,
                                const mla_cache* cache, const int32_t* seq_lens, int32_t batch,
                                int32_t s_q, int32_t causal, int32_t n_split, void* workspace,
                                size_t workspace_bytes, void* o_lat, float* lse, void* stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if (batch < 0 || s_q <= 0 || n_split < 0 || (causal != 0 && causal != 1)) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if ((s = check_cache(dims, cache)) != MLA_OK) return s;
  if (!q_packed || !seq_lens || !o_lat) return MLA_ERR_INVALID_ARG;
  if (batch > cache->num_seqs) return MLA_ERR_INVALID_ARG;
  if (dims->d_c + dims->d_rope > 576 || dims->d_c > 512 || dims->d_c % 4) return MLA_ERR_UNSUPPORTED;
  const bool planned = partitioned(dims);
  const int n = planned ? 0 : effective_split(dims, batch, s_q, n_split, cache->max_pages_per_seq);
  size_t need = mla_decode_workspace_size(dims, batch, s_q, n_split, cache->max_pages_per_seq);
  if (need > 0 && (workspace_bytes < need || !workspace)) return MLA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (!err) return MLA_ERR_CUDA;
  DecodeArgs a;
  a.q = q_packed;
  a.cache = make_view(dims, cache);
  a.seq_lens = seq_lens;
  a.batch = batch;
  a.s_q = s_q;
  a.causal = causal;
  a.n_split = n;
  a.n_heads = dims->n_heads;
  a.d_c = dims->d_c;
  a.d_rope = dims->d_rope;
  a.act = dims->act_dtype;
  a.scale = dims->scale;
  a.plan = planned ? 1 : 0;
  a.rowinfo = nullptr;
  if (planned) {
    const size_t slots = (size_t)(decode_path(dims) == DecodePath::SmallHead ? SH_PLAN_SLOTS : TC_PLAN_SLOTS);
    a.o_part = static_cast<float*>(workspace);
    a.lse_part = a.o_part + slots * dims->n_heads * dims->d_c;
    a.rowinfo = reinterpret_cast<int32_t*>(a.lse_part + slots * dims->n_heads);
  } else {
    size_t rows = (size_t)batch * n * s_q * dims->n_heads;
    a.o_part = n > 1 ? static_cast<float*>(workspace) : nullptr;
    a.lse_part = n > 1 ? static_cast<float*>(workspace) + rows * dims->d_c : nullptr;
  }
  a.o_lat = o_lat;
  a.lse = lse;
  a.err = err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the partitioned launchers run their own combine
  const DecodePath path = decode_path(dims);
  cudaError_t e = path == DecodePath::SmallHead    ? launch_decode_sh(a, st)
                  : path == DecodePath::TensorCore ? launch_decode_tc(a, st)
                                                   : launch_decode_simt(a, st);
  if (e != cudaSuccess) return cuda_status(e);
  if (!planned && n > 1) e = launch_combine(a, st);
  return cuda_status(e);
}

mla_status mla_output_up(const mla_dims* dims, const void* o_lat, int32_t n_tok,
                         const void* w_uv, void* out, void* stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!o_lat || !w_uv || !out) return MLA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (!err) return MLA_ERR_CUDA;
  return cuda_status(launch_output_up(*dims, o_lat, n_tok, w_uv, out, err, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
