// mea_internal.h -- launch descriptions shared between the C-ABI translation unit
// and the kernel translation units (host side only; no kernel code here).
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stdint.h>

#include <atomic>

namespace mea {

// Raises kernel KERN's dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute lasts as long as the device's
// context); later calls only test a bit.  If the context is destroyed and
// created again (cudaDeviceReset), the bit stays set and the kernel's launch
// then fails with an error status instead of running.
template <auto KERN>
cudaError_t set_smem_once(int bytes) {
  static std::atomic<unsigned long long> done{0};  // bit d: done on device d (d < 64)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Prefill: one CTA computes two 128-row query tiles of one (sequence, head).
constexpr int kFwdRowsPerCta = 256;

struct FwdArgs {
  void* out;
  float* lse;                  // [B, Hq, M] or nullptr
  const int32_t* seqstart_q;   // packed batches only
  const int32_t* seqstart_k;
  int* status;                 // device status word
  long long o_sb, o_sm, o_sh;  // out strides (elements)
  int B, M, N, Hq, Hkv, group;
  int num_units;    // B for dense batches, num_seqs for packed ones
  int num_mblocks;  // ceil(max query rows per unit / kFwdRowsPerCta)
  float scale_log2; // scale * log2(e)
  // Block-sparse only (nullptr otherwise): byte [b * bm_sb + h * bm_sh +
  // (query row / 128) * bm_nk + key / 128], zero = block left out.
  const uint8_t* block_mask;
  long long bm_sb, bm_sh;
  int bm_nk;        // ceil(N / 128)
  // Prefill chunk against a cache only (cache_len nullptr otherwise): the
  // chunk's q/out/lse have M rows per sequence, of which q_lens[b] (nullptr: M)
  // are real; the caches [B, cap, Hkv, K] hold cache_len[b] rows before the call.
  const int32_t* cache_len;
  const int32_t* q_lens;
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  long long kn_s[3], vn_s[3], kc_s[3], vc_s[3];  // element strides (b, row, head)
  int cap;
};

constexpr int kSparseBlock = 128;  // rows and keys per block-mask entry

struct FwdLaunch {
  CUtensorMap tmQ, tmK, tmV;
  CUtensorMap tmKn, tmVn;  // new keys / values of a prefill chunk (cache mode only)
  FwdArgs args;
  int head_dim;   // 64 or 128
  bool bf16;
  int mask;       // mea_bias_t value
  bool alibi;
};

cudaError_t launch_fwd(const FwdLaunch& launch, cudaStream_t stream);

// Rows with no visible key (or an empty key set): out = 0, lse = -inf.
cudaError_t launch_fill_empty(void* out, float* lse, int B, int M, int Hq, int K, long long o_sb,
                              long long o_sm, long long o_sh, cudaStream_t stream);

// Decode: split-KV partial kernel + log-sum-exp merge.
constexpr int kDecodeChunk = 512;  // cache rows per split

struct DecodeArgs {
  const void* q;               // [B, Hq, K]
  void* out;                   // [B, Hq, K]
  float* lse;                  // [B, Hq] or nullptr
  const int32_t* kv_seqstart;  // [B + 1]
  float* part_o;               // [B, Hq, max_splits, K]
  float* part_lse;             // [B, Hq, max_splits] (log2 domain)
  int* status;
  int B, Hq, Hkv, group, max_splits, cache_rows;
  float scale_log2;
};

struct DecodeLaunch {
  CUtensorMap tmK, tmV;
  DecodeArgs args;
  int head_dim;
  bool bf16;
  bool alibi;
};

cudaError_t launch_decode(const DecodeLaunch& launch, cudaStream_t stream);

// Backward: dq, dk, dv from q, k, v, out, dout and the forward's lse.
constexpr int kBwdBlock = 128;  // keys per CTA

struct BwdArgs {
  const void *q, *k, *v, *out, *dout;  // contiguous [B,M,Hq,K] / [B,N,Hkv,K]
  const float* lse;                    // [B, Hq, M] natural log (from mea_fwd)
  void *dq, *dk, *dv;
  float* dq_acc;                       // [B, M, Hq, K] fp32 workspace
  float* delta;                        // [B, Hq, M] fp32 workspace: <dout_i, out_i>
  const int32_t* seqstart_q;
  const int32_t* seqstart_k;
  int* status;
  int B, M, N, Hq, Hkv, group, num_units, num_kblocks;
  float scale, scale_log2;
};

struct BwdLaunch {
  CUtensorMap tmQ, tmK, tmV, tmDO;  // boxes: bwd_query_block rows (q, dout), kBwdBlock rows (k, v)
  CUtensorMap tmDQ;                 // fp32 dq accumulator, 32 x 1 x bwd_dq_box_rows boxes
  BwdArgs args;
  int head_dim;
  bool bf16;
  int mask;
  bool alibi;
};

// stages: bit 0 the D / accumulator preparation, bit 1 the main kernel, bit 2
// the dq conversion (the three launches of one backward, in that order).
cudaError_t launch_bwd(const BwdLaunch& launch, cudaStream_t stream, int stages = 7);

// Query rows per step of the backward kernel for head dimension 64 or 128.
int bwd_query_block(int head_dim);
int bwd_dq_box_rows(int head_dim);  // rows of the dq accumulator's TMA reduction boxes

}  // namespace mea
