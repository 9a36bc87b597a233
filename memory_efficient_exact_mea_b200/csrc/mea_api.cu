// mea_api.cu -- the C ABI declared in include/mea.h: host-side validation,
// TMA descriptor encoding and kernel dispatch.  No allocation, no global mutable
// host state (the driver entry point is resolved once, thread-safely).
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "mea.h"
#include "mea_internal.h"
#include "sm100.cuh"

// First error recorded by a kernel of this library (one word per device).
__device__ int g_mea_status = 0;

namespace {

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int* status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_mea_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A [batch, rows, heads, K] tensor with element strides {sb, sm, sh} as a rank-4
// TMA map (innermost first), 64-element x 1 head x `box_rows` boxes, 128-byte
// swizzle.  Returns false if the driver rejects it.
bool encode_bmhk(CUtensorMap* map, const void* base, bool bf16, int batch, int rows, int heads,
                 int K, const int64_t st[3], int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(st[2]) * 2,
                                 static_cast<cuuint64_t>(st[1]) * 2,
                                 static_cast<cuuint64_t>(st[0]) * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A contiguous fp32 [batch, rows, heads, K] tensor as a rank-4 TMA map with
// 32-element x 1 head x `box_rows` boxes and 128-byte swizzle (reduction target).
bool encode_f32_bmhk(CUtensorMap* map, void* base, int batch, int rows, int heads, int K,
                     int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(K) * 4,
                                 static_cast<cuuint64_t>(heads) * K * 4,
                                 static_cast<cuuint64_t>(rows) * heads * K * 4};
  const cuuint32_t box[4] = {32, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A packed cache [rows, heads, K] (contiguous) as a rank-3 TMA map.
bool encode_cache(CUtensorMap* map, const void* base, bool bf16, int rows, int heads, int K,
                  int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2,
                                 static_cast<cuuint64_t>(heads) * K * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool strides_ok(const int64_t s[3]) {
  for (int i = 0; i < 3; ++i)
    if (s[i] <= 0 || (s[i] & 7) != 0 || s[i] >= (int64_t(1) << 38)) return false;
  return true;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int decode_splits(int max_kv_len) {
  return max_kv_len <= 0 ? 0 : (max_kv_len + mea::kDecodeChunk - 1) / mea::kDecodeChunk;
}

}  // namespace

extern "C" {

int mea_version(void) { return kVersion; }

const char* mea_status_string(int status) {
  switch (status) {
    case MEA_OK: return "ok";
    case MEA_ERR_INVALID_ARG: return "invalid argument";
    case MEA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MEA_ERR_WORKSPACE: return "workspace missing or too small";
    case MEA_ERR_CUDA: return "CUDA error";
    case MEA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int mea_decode_chunk(void) { return mea::kDecodeChunk; }

// mea_fwd and mea_fwd_block_sparse (block_mask != nullptr: bias none or causal,
// mask_strides = element strides of the mask for b and h).
static int fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                    int M, int N, int Hq, int Hkv, int K, const int64_t q_strides[3],
                    const int64_t k_strides[3], const int64_t v_strides[3],
                    const int64_t o_strides[3], mea_dtype_t dtype, mea_bias_t bias,
                    const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
                    int max_seqlen_q, int alibi, float scale, const uint8_t* block_mask,
                    const int64_t* mask_strides, cudaStream_t stream) {
  if (B < 0 || M < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return MEA_ERR_INVALID_ARG;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_INVALID_ARG;
  if (bias < MEA_BIAS_NONE || bias > MEA_BIAS_BLOCKDIAG_CAUSAL) return MEA_ERR_INVALID_ARG;
  if (!q_strides || !k_strides || !v_strides || !o_strides) return MEA_ERR_INVALID_ARG;
  if (!(scale == scale)) return MEA_ERR_INVALID_ARG;  // NaN
  if (B == 0 || M == 0) return MEA_OK;
  if (!q || !out || (N > 0 && (!k || !v))) return MEA_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return MEA_ERR_UNSUPPORTED;
  if (scale < 0.f) return MEA_ERR_UNSUPPORTED;  // the kernel takes row maxima on raw scores
  const bool packed = bias == MEA_BIAS_BLOCKDIAG || bias == MEA_BIAS_BLOCKDIAG_CAUSAL;
  if (packed) {
    if (B != 1 || !seqstart_q || num_seqs <= 0 || max_seqlen_q < 0) return MEA_ERR_INVALID_ARG;
    if (!seqstart_k && M != N) return MEA_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(out) || (N > 0 && (!aligned16(k) || !aligned16(v))))
    return MEA_ERR_UNSUPPORTED;
  if (!strides_ok(q_strides) || !strides_ok(o_strides) ||
      (N > 0 && (!strides_ok(k_strides) || !strides_ok(v_strides))))
    return MEA_ERR_UNSUPPORTED;

  int* status = status_word();
  if (!status) return MEA_ERR_CUDA;

  if (N == 0) {  // no key anywhere: every row is empty
    return mea::launch_fill_empty(out, lse, B, M, Hq, K, o_strides[0], o_strides[1],
                                  o_strides[2], stream) == cudaSuccess
               ? MEA_OK
               : MEA_ERR_CUDA;
  }

  mea::FwdLaunch L{};
  const bool bf16 = dtype == MEA_BF16;
  if (!encode_bmhk(&L.tmQ, q, bf16, B, M, Hq, K, q_strides, 128) ||
      !encode_bmhk(&L.tmK, k, bf16, B, N, Hkv, K, k_strides, 128) ||
      !encode_bmhk(&L.tmV, v, bf16, B, N, Hkv, K, v_strides, 128))
    return MEA_ERR_CUDA;
  mea::FwdArgs& a = L.args;
  a.out = out;
  a.lse = lse;
  a.seqstart_q = packed ? seqstart_q : nullptr;
  a.seqstart_k = packed ? (seqstart_k ? seqstart_k : seqstart_q) : nullptr;
  a.status = status;
  a.o_sb = o_strides[0];
  a.o_sm = o_strides[1];
  a.o_sh = o_strides[2];
  a.B = B;
  a.M = M;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.group = Hq / Hkv;
  a.num_units = packed ? num_seqs : B;
  const int rows = packed ? max_seqlen_q : M;
  a.num_mblocks = (rows + mea::kFwdRowsPerCta - 1) / mea::kFwdRowsPerCta;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.block_mask = block_mask;
  if (block_mask) {
    a.bm_sb = mask_strides[0];
    a.bm_sh = mask_strides[1];
    a.bm_nk = (N + mea::kSparseBlock - 1) / mea::kSparseBlock;
  }
  L.head_dim = K;
  L.bf16 = bf16;
  L.mask = static_cast<int>(bias);
  L.alibi = alibi != 0;
  if (a.num_mblocks == 0) return MEA_OK;
  return mea::launch_fwd(L, stream) == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

int mea_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int M,
            int N, int Hq, int Hkv, int K, const int64_t q_strides[3], const int64_t k_strides[3],
            const int64_t v_strides[3], const int64_t o_strides[3], mea_dtype_t dtype,
            mea_bias_t bias, const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
            int max_seqlen_q, int max_seqlen_k, int alibi, float scale, cudaStream_t stream) {
  (void)max_seqlen_k;
  return fwd_impl(q, k, v, out, lse, B, M, N, Hq, Hkv, K, q_strides, k_strides, v_strides,
                  o_strides, dtype, bias, seqstart_q, seqstart_k, num_seqs, max_seqlen_q, alibi,
                  scale, nullptr, nullptr, stream);
}

int mea_sparse_block_size(void) { return mea::kSparseBlock; }

int mea_prefill_chunk(const void* q, const void* k_new, const void* v_new, void* k_cache,
                      void* v_cache, const int32_t* cache_seqlens, const int32_t* q_seqlens,
                      void* out, float* lse, int B, int M, int cache_rows, int Hq, int Hkv,
                      int K, const int64_t q_strides[3], const int64_t kn_strides[3],
                      const int64_t vn_strides[3], const int64_t kc_strides[3],
                      const int64_t vc_strides[3], const int64_t o_strides[3],
                      mea_dtype_t dtype, int causal, int alibi, float scale,
                      cudaStream_t stream) {
  if (B < 0 || M < 0 || cache_rows < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
    return MEA_ERR_INVALID_ARG;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return MEA_ERR_INVALID_ARG;
  if (!q_strides || !kn_strides || !vn_strides || !kc_strides || !vc_strides || !o_strides)
    return MEA_ERR_INVALID_ARG;
  if (!(scale == scale)) return MEA_ERR_INVALID_ARG;
  if (B == 0 || M == 0) return MEA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_seqlens || !out)
    return MEA_ERR_INVALID_ARG;
  if (cache_rows < 1) return MEA_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return MEA_ERR_UNSUPPORTED;
  if (scale < 0.f) return MEA_ERR_UNSUPPORTED;
  for (const void* p : {q, k_new, v_new, static_cast<const void*>(k_cache),
                        static_cast<const void*>(v_cache), static_cast<const void*>(out)})
    if (!aligned16(p)) return MEA_ERR_UNSUPPORTED;
  for (const int64_t* st : {q_strides, kn_strides, vn_strides, kc_strides, vc_strides, o_strides})
    if (!strides_ok(st)) return MEA_ERR_UNSUPPORTED;
  int* status = status_word();
  if (!status) return MEA_ERR_CUDA;

  mea::FwdLaunch L{};
  const bool bf16 = dtype == MEA_BF16;
  if (!encode_bmhk(&L.tmQ, q, bf16, B, M, Hq, K, q_strides, 128) ||
      !encode_bmhk(&L.tmK, k_cache, bf16, B, cache_rows, Hkv, K, kc_strides, 128) ||
      !encode_bmhk(&L.tmV, v_cache, bf16, B, cache_rows, Hkv, K, vc_strides, 128) ||
      !encode_bmhk(&L.tmKn, k_new, bf16, B, M, Hkv, K, kn_strides, 128) ||
      !encode_bmhk(&L.tmVn, v_new, bf16, B, M, Hkv, K, vn_strides, 128))
    return MEA_ERR_CUDA;
  mea::FwdArgs& a = L.args;
  a.out = out;
  a.lse = lse;
  a.status = status;
  a.o_sb = o_strides[0];
  a.o_sm = o_strides[1];
  a.o_sh = o_strides[2];
  a.B = B;
  a.M = M;
  a.N = cache_rows;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.group = Hq / Hkv;
  a.num_units = B;
  a.num_mblocks = (M + mea::kFwdRowsPerCta - 1) / mea::kFwdRowsPerCta;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.cache_len = cache_seqlens;
  a.q_lens = q_seqlens;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  for (int i = 0; i < 3; ++i) {
    a.kn_s[i] = kn_strides[i];
    a.vn_s[i] = vn_strides[i];
    a.kc_s[i] = kc_strides[i];
    a.vc_s[i] = vc_strides[i];
  }
  a.cap = cache_rows;
  L.head_dim = K;
  L.bf16 = bf16;
  L.mask = causal ? static_cast<int>(MEA_BIAS_CAUSAL) : static_cast<int>(MEA_BIAS_NONE);
  L.alibi = alibi != 0;
  return mea::launch_fwd(L, stream) == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

int mea_fwd_block_sparse(const void* q, const void* k, const void* v, void* out, float* lse,
                         int B, int M, int N, int Hq, int Hkv, int K,
                         const int64_t q_strides[3], const int64_t k_strides[3],
                         const int64_t v_strides[3], const int64_t o_strides[3],
                         mea_dtype_t dtype, mea_bias_t bias, const uint8_t* block_mask,
                         const int64_t mask_strides[2], int alibi, float scale,
                         cudaStream_t stream) {
  if (bias != MEA_BIAS_NONE && bias != MEA_BIAS_CAUSAL) {
    if (bias < MEA_BIAS_NONE || bias > MEA_BIAS_BLOCKDIAG_CAUSAL) return MEA_ERR_INVALID_ARG;
    return MEA_ERR_UNSUPPORTED;
  }
  if (!mask_strides || mask_strides[0] < 0 || mask_strides[1] < 0) return MEA_ERR_INVALID_ARG;
  if (B > 0 && M > 0 && N > 0 && !block_mask) return MEA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, out, lse, B, M, N, Hq, Hkv, K, q_strides, k_strides, v_strides,
                  o_strides, dtype, bias, nullptr, nullptr, 0, 0, alibi, scale,
                  N > 0 ? block_mask : nullptr, mask_strides, stream);
}

size_t mea_decode_workspace_size(int B, int Hq, int Hkv, int K, int max_kv_len) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || K <= 0 || max_kv_len < 0) return 0;
  const size_t splits = static_cast<size_t>(decode_splits(max_kv_len));
  const size_t rows = static_cast<size_t>(B) * Hq * splits;
  return align256(rows * K * sizeof(float)) + align256(rows * sizeof(float));
}

int mea_decode(const void* q, const void* k_cache, const void* v_cache,
               const int32_t* kv_seqstart, void* out, float* lse, int B, int Hq, int Hkv, int K,
               int cache_rows, int max_kv_len, mea_dtype_t dtype, int alibi, float scale,
               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || cache_rows < 0 || max_kv_len < 0)
    return MEA_ERR_INVALID_ARG;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_INVALID_ARG;
  if (!(scale == scale)) return MEA_ERR_INVALID_ARG;
  if (B == 0) return MEA_OK;
  if (!q || !out || !kv_seqstart) return MEA_ERR_INVALID_ARG;
  if (cache_rows > 0 && (!k_cache || !v_cache)) return MEA_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return MEA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return MEA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) ||
      (cache_rows > 0 && (!aligned16(k_cache) || !aligned16(v_cache))))
    return MEA_ERR_UNSUPPORTED;
  const size_t need = mea_decode_workspace_size(B, Hq, Hkv, K, max_kv_len);
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return MEA_ERR_WORKSPACE;

  int* status = status_word();
  if (!status) return MEA_ERR_CUDA;

  mea::DecodeLaunch L{};
  const bool bf16 = dtype == MEA_BF16;
  mea::DecodeArgs& a = L.args;
  a.q = q;
  a.out = out;
  a.lse = lse;
  a.kv_seqstart = kv_seqstart;
  a.status = status;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.group = Hq / Hkv;
  a.cache_rows = cache_rows;
  a.max_splits = cache_rows > 0 ? decode_splits(max_kv_len) : 0;
  const size_t rows = static_cast<size_t>(B) * Hq * decode_splits(max_kv_len);
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                        align256(rows * K * sizeof(float)));
  a.scale_log2 = scale * 1.4426950408889634f;
  L.head_dim = K;
  L.bf16 = bf16;
  L.alibi = alibi != 0;
  if (a.max_splits > 0) {
    if (!encode_cache(&L.tmK, k_cache, bf16, cache_rows, Hkv, K, 64) ||
        !encode_cache(&L.tmV, v_cache, bf16, cache_rows, Hkv, K, 64))
      return MEA_ERR_CUDA;
  }
  return mea::launch_decode(L, stream) == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

int mea_read_device_status(cudaStream_t stream, int clear) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MEA_ERR_CUDA;
  int value = 0;
  if (cudaMemcpyFromSymbol(&value, g_mea_status, sizeof(int)) != cudaSuccess)
    return MEA_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_mea_status, &zero, sizeof(int)) != cudaSuccess) return MEA_ERR_CUDA;
  }
  return value;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Failure-path self-test: one CTA waits on an mbarrier that nothing will ever
// arrive on, through the same bounded wait the kernels use, with a short limit.
// ---------------------------------------------------------------------------
namespace {

__global__ void selftest_timeout_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mea::mbar_init(&bar, 1);
    abort_flag = 0;
    mea::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mea::mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
}

}  // namespace

extern "C" int mea_selftest_timeout(int timeout_us, cudaStream_t stream) {
  if (timeout_us <= 0 || timeout_us > 10000000) return MEA_ERR_INVALID_ARG;
  int* status = status_word();
  if (!status) return MEA_ERR_CUDA;
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(status, 1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
extern "C" size_t mea_bwd_workspace_size(int B, int M, int Hq, int K) {
  if (B < 0 || M < 0 || Hq <= 0 || K <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * M * Hq;
  return align256(rows * K * sizeof(float)) + align256(rows * sizeof(float));
}

extern "C" int mea_bwd_stages(const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int M, int N, int Hq, int Hkv, int K, mea_dtype_t dtype,
                              mea_bias_t bias, const int32_t* seqstart_q,
                              const int32_t* seqstart_k, int num_seqs, int max_seqlen_q,
                              int max_seqlen_k, int alibi, float scale, void* workspace,
                              size_t workspace_bytes, int stages, cudaStream_t stream) {
  (void)max_seqlen_q;
  if (stages <= 0 || stages > 7) return MEA_ERR_INVALID_ARG;
  if (B < 0 || M < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return MEA_ERR_INVALID_ARG;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_INVALID_ARG;
  if (bias < MEA_BIAS_NONE || bias > MEA_BIAS_BLOCKDIAG_CAUSAL) return MEA_ERR_INVALID_ARG;
  if (!(scale == scale)) return MEA_ERR_INVALID_ARG;
  if (B == 0 || (M == 0 && N == 0)) return MEA_OK;
  if ((M > 0 && (!q || !out || !dout || !lse || !dq)) || (N > 0 && (!k || !v || !dk || !dv)))
    return MEA_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return MEA_ERR_UNSUPPORTED;
  const bool packed = bias == MEA_BIAS_BLOCKDIAG || bias == MEA_BIAS_BLOCKDIAG_CAUSAL;
  if (packed) {
    if (B != 1 || !seqstart_q || num_seqs <= 0 || max_seqlen_k < 0) return MEA_ERR_INVALID_ARG;
    if (!seqstart_k && M != N) return MEA_ERR_INVALID_ARG;
  }
  for (const void* p : {q, k, v, out, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if (p && !aligned16(p)) return MEA_ERR_UNSUPPORTED;
  const size_t need = mea_bwd_workspace_size(B, M, Hq, K);
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return MEA_ERR_WORKSPACE;
  int* status = status_word();
  if (!status) return MEA_ERR_CUDA;

  mea::BwdLaunch L{};
  const bool bf16 = dtype == MEA_BF16;
  if (M > 0 && N > 0) {
    const int64_t sq[3] = {static_cast<int64_t>(M) * Hq * K, static_cast<int64_t>(Hq) * K, K};
    const int64_t sk[3] = {static_cast<int64_t>(N) * Hkv * K, static_cast<int64_t>(Hkv) * K, K};
    const int bm = mea::bwd_query_block(K);
    if (!encode_bmhk(&L.tmQ, q, bf16, B, M, Hq, K, sq, bm) ||
        !encode_bmhk(&L.tmDO, dout, bf16, B, M, Hq, K, sq, bm) ||
        !encode_bmhk(&L.tmK, k, bf16, B, N, Hkv, K, sk, mea::kBwdBlock) ||
        !encode_bmhk(&L.tmV, v, bf16, B, N, Hkv, K, sk, mea::kBwdBlock) ||
        !encode_f32_bmhk(&L.tmDQ, workspace, B, M, Hq, K, mea::bwd_dq_box_rows(K)))
      return MEA_ERR_CUDA;
  }
  mea::BwdArgs& a = L.args;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  const size_t rows = static_cast<size_t>(B) * M * Hq;
  a.dq_acc = static_cast<float*>(workspace);
  a.delta = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                     align256(rows * K * sizeof(float)));
  a.seqstart_q = packed ? seqstart_q : nullptr;
  a.seqstart_k = packed ? (seqstart_k ? seqstart_k : seqstart_q) : nullptr;
  a.status = status;
  a.B = B;
  a.M = M;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.group = Hq / Hkv;
  a.num_units = packed ? num_seqs : B;
  const int krows = packed ? max_seqlen_k : N;
  a.num_kblocks = (krows + mea::kBwdBlock - 1) / mea::kBwdBlock;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  L.head_dim = K;
  L.bf16 = bf16;
  L.mask = static_cast<int>(bias);
  L.alibi = alibi != 0;
  // The kernel writes every key row of every sequence; rows no sequence owns
  // (packed batches) and the no-query case are zeroed here (with the main stage).
  if ((stages & MEA_BWD_MAIN) && N > 0 && (M == 0 || packed) &&
      (cudaMemsetAsync(dk, 0, static_cast<size_t>(B) * N * Hkv * K * 2, stream) != cudaSuccess ||
       cudaMemsetAsync(dv, 0, static_cast<size_t>(B) * N * Hkv * K * 2, stream) != cudaSuccess))
    return MEA_ERR_CUDA;
  if (M == 0) return MEA_OK;
  return mea::launch_bwd(L, stream, stages) == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

extern "C" int mea_bwd(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int M, int N, int Hq, int Hkv, int K, mea_dtype_t dtype, mea_bias_t bias,
                       const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
                       int max_seqlen_q, int max_seqlen_k, int alibi, float scale,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return mea_bwd_stages(q, k, v, out, dout, lse, dq, dk, dv, B, M, N, Hq, Hkv, K, dtype, bias,
                        seqstart_q, seqstart_k, num_seqs, max_seqlen_q, max_seqlen_k, alibi,
                        scale, workspace, workspace_bytes,
                        MEA_BWD_PREP | MEA_BWD_MAIN | MEA_BWD_DQ, stream);
}
