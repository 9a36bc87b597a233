// mea_bwd_sm100.cu -- attention backward on B200 (sm_100a): TMA + tcgen05 + TMEM.
//
// The backward pass recomputes the attention weights from q, k and the
// forward's log-sum-exp instead of storing them ("FlashAttention (2022)",
// section "Il trucco della softmax che non ha bisogno di vedere tutto").  With
// D_i = <dO_i, O_i> and p_ij = exp(s_ij - lse_i):
//     dV_j = sum_i p_ij dO_i          dP_ij = <dO_i, v_j>
//     dS_ij = p_ij (dP_ij - D_i)      dQ_i = scale sum_j dS_ij k_j
//     dK_j = scale sum_i dS_ij q_i    (dK, dV summed over the query heads of a kv head)
//
// Three kernels:
//   bwd_prep     D_i for every row, and a zeroed fp32 dq accumulator;
//   bwd_kernel   one CTA per (128-key block, kv head, batch or sequence): K_j, V_j
//                stay in shared memory and dK_j, dV_j accumulate in tensor memory
//                while the CTA walks the query heads of the group and the query
//                blocks that can see its keys;
//   bwd_dq_out   dq accumulator -> fp16/bf16.
//
// bwd_kernel, per query block i of BM rows (BM = 64 at K = 128, 128 at K = 64),
// with the block's keys on the 128 TMEM lanes:
//   S^T  = K Q_i^T,  dP^T = V dO_i^T                  (tcgen05, both operands K-major)
//   P^T, dS^T from S^T, dP^T, lse_i, D_i               (128 threads, one per key)
//     P^T (16-bit) is written back over S^T in TMEM, dS^T to shared memory
//   dV  += P^T dO_i   (A = P^T from TMEM)              dK += dS^T Q_i
//   dQ_i = dS_i K  (K = 64)  or  dQ_i^T = K^T dS_i^T (K = 128): both M = 128, N = 64
//   dQ_i is drained by four warps into the fp32 accumulator with global reductions.
// TMEM columns: S^T [0, BM) | dP^T [BM, 2BM) | dQ [2BM, 2BM+64) | dV (K) | dK (K).
//
// CTA (320 threads): warps 0-3 P/dS and the dK/dV epilogue, warps 4-7 the dQ
// drain, warp 8 allocates TMEM and one of its threads issues every MMA, warp 9
// loads (one thread issues the TMA copies; the warp stages lse and D of each block).
#include <math.h>

#include <algorithm>

#include "mea_internal.h"
#include "sm100.cuh"

namespace mea {
namespace {

constexpr int kBN = kBwdBlock;  // keys per CTA (= TMEM lanes)
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }
__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

template <bool BF16>
__device__ __forceinline__ float to_f(uint16_t x) {
  if constexpr (BF16) return __uint_as_float(static_cast<uint32_t>(x) << 16);
  else return __half2float(__ushort_as_half(x));
}

template <int D>
struct BwdCfg {
  static constexpr int BM = (D == 128) ? 64 : 128;  // query rows per step
  static constexpr int kChunksD = D / 64;           // 64-element column chunks of a K-wide row
  static constexpr int kKVChunk = kBN * 128;        // one chunk of a 128-row tile
  static constexpr int kQChunk = BM * 128;          // one chunk of a BM-row tile
  static constexpr int kKVTile = kChunksD * kKVChunk;
  static constexpr int kQTile = kChunksD * kQChunk;
  static constexpr int kDSTile = (BM / 64) * kKVChunk;  // dS^T: 128 keys x BM queries
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int kK = 0;
  static constexpr int kV = kKVTile;
  static constexpr int kQ = 2 * kKVTile;              // two stages
  static constexpr int kDO = kQ + 2 * kQTile;         // two stages
  static constexpr int kDS = kDO + 2 * kQTile;
  static constexpr int kLse = kDS + kDSTile;          // [2][BM] lse * log2(e) (+inf: no weight)
  static constexpr int kDelta = kLse + 2 * BM * 4;    // [2][BM]
  static constexpr int kBar = kDelta + 2 * BM * 4;
  static constexpr int kNumBars = 10;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;
  // tensor memory columns
  static constexpr uint32_t kColS = 0, kColDP = BM, kColDQ = 2 * BM, kColDV = 2 * BM + 64,
                            kColDK = 2 * BM + 64 + D;
  static_assert(kColDK + D <= kTmemCols, "tensor memory layout");
};

// One warp per (row, query head): D = <dout, out>, and zero the dq accumulator row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.M * a.Hq;
  if (row >= rows) return;
  const long long b = row / (static_cast<long long>(a.M) * a.Hq);
  const long long i = (row / a.Hq) % a.M;
  const long long h = row % a.Hq;
  const uint16_t* o = static_cast<const uint16_t*>(a.out) + row * D;
  const uint16_t* g = static_cast<const uint16_t*>(a.dout) + row * D;
  float s = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) s = fmaf(to_f<BF16>(o[d]), to_f<BF16>(g[d]), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) a.delta[(b * a.Hq + h) * a.M + i] = s;
#pragma unroll
  for (int d = lane; d < D; d += 32) a.dq_acc[row * D + d] = 0.f;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_dq_out_kernel(const BwdArgs a) {
  const long long n = static_cast<long long>(a.B) * a.M * a.Hq * D / 2;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float2 v = reinterpret_cast<const float2*>(a.dq_acc)[e];
    reinterpret_cast<uint32_t*>(a.dq)[e] = pack2<BF16>(v.x, v.y);
  }
}

template <int D, bool BF16, int MASK, bool ALIBI>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const BwdArgs a) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM;
  constexpr bool kCausal = (MASK == 1 || MASK == 3);
  constexpr bool kPacked = (MASK >= 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;    // [2] Q, dO (+ lse, D) of a step landed
  uint64_t* q_empty = bars + 3;   // [2] every MMA reading the stage completed
  uint64_t* s_full = bars + 5;    // S^T, dP^T of the step are in TMEM
  uint64_t* p_ready = bars + 6;   // P^T in TMEM and dS^T in shared memory (128 arrivals)
  uint64_t* dq_full = bars + 7;   // dQ of the step is in TMEM
  uint64_t* dq_empty = bars + 8;  // dQ read out of TMEM (128 arrivals)
  uint64_t* mma_done = bars + 9;
  float* s_lse = reinterpret_cast<float*>(smem + C::kLse);
  float* s_delta = reinterpret_cast<float*>(smem + C::kDelta);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = blockIdx.x, kvh = blockIdx.y, unit = blockIdx.z;

  int q0 = 0, q_len = a.M, k0 = 0, k_len = a.N, bidx = unit;
  if constexpr (kPacked) {
    q0 = a.seqstart_q[unit];
    q_len = a.seqstart_q[unit + 1] - q0;
    k0 = a.seqstart_k[unit];
    k_len = a.seqstart_k[unit + 1] - k0;
    bidx = 0;
    if (q_len < 0 || k_len < 0 || q0 < 0 || k0 < 0 || q0 + q_len > a.M || k0 + k_len > a.N ||
        (nb == a.num_kblocks - 1 && k_len > a.num_kblocks * kBN)) {
      if (threadIdx.x == 0) record_error(a.status, kErrInvalidArg);
      return;
    }
  }
  const int n0 = nb * kBN;
  if (n0 >= k_len) return;
  const int off = k_len - q_len;  // bottom-right causal alignment
  // First query block whose rows can see a key of this block.
  int m_first = 0;
  if constexpr (kCausal) m_first = max(0, n0 - off) / BM * BM;
  const int n_mblocks = q_len > m_first ? (q_len - m_first + BM - 1) / BM : 0;
  const int steps = a.group * n_mblocks;  // (query head, query block) pairs, head-major

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, 128);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kLoadWarp) {
    // ===================== loads =============================================
    bool ok = true;
    int issued = 0;
    if (lane == 0 && steps > 0) {
      mbar_arrive_expect_tx(kv_full, 2 * C::kKVTile);
      for (int c = 0; c < C::kChunksD; ++c) {
        tma_load_4d(smem + C::kK + c * C::kKVChunk, &tmK, kv_full, c * 64, kvh, k0 + n0, bidx);
        tma_load_4d(smem + C::kV + c * C::kKVChunk, &tmV, kv_full, c * 64, kvh, k0 + n0, bidx);
      }
    }
    for (int s = 0; s < steps && ok; ++s) {
      const int h = kvh * a.group + s / n_mblocks;
      const int m0 = m_first + (s % n_mblocks) * BM;
      const int slot = s & 1;
      if (!(ok = mbar_wait_warp(&q_empty[slot], ((s >> 1) & 1) ^ 1, abort_flag, a.status))) break;
      // lse (log2 units) and D of the block's rows; +inf marks a row that takes
      // no weight (past the sequence, or no visible key in the forward).
      for (int r = lane; r < BM; r += 32) {
        const int i = m0 + r;
        float l2 = pos_inf(), dl = 0.f;
        if (i < q_len) {
          const long long li = (static_cast<long long>(bidx) * a.Hq + h) * a.M + q0 + i;
          const float l = a.lse[li];
          if (l != neg_inf()) l2 = l * kLog2e;
          dl = a.delta[li];
        }
        s_lse[slot * BM + r] = l2;
        s_delta[slot * BM + r] = dl;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[slot], 2 * C::kQTile);
        for (int c = 0; c < C::kChunksD; ++c) {
          tma_load_4d(smem + C::kQ + slot * C::kQTile + c * C::kQChunk, &tmQ, &q_full[slot],
                      c * 64, h, q0 + m0, bidx);
          tma_load_4d(smem + C::kDO + slot * C::kQTile + c * C::kQChunk, &tmDO, &q_full[slot],
                      c * 64, h, q0 + m0, bidx);
        }
      }
      issued = s + 1;
    }
    // Let every copy this warp started land before the CTA can exit.
    if (lane == 0 && steps > 0) {
      mbar_wait_drain(kv_full, 0, a.status);
      for (int s = max(0, issued - 2); s < issued; ++s)
        mbar_wait_drain(&q_full[s & 1], (s >> 1) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ===================== MMA issue (one thread) ============================
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_ab(BF16, kBN, BM, false, false);
      constexpr uint32_t idesc_g = idesc_f16_ab(BF16, kBN, D, false, true);
      constexpr uint32_t idesc_q = idesc_f16_ab(BF16, kBN, 64, true, true);
      const uint32_t sK = smem_u32(smem + C::kK), sV = smem_u32(smem + C::kV);
      const uint32_t sDS = smem_u32(smem + C::kDS);
      const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP;
      const uint32_t tDQ = tmem_base + C::kColDQ, tDV = tmem_base + C::kColDV;
      const uint32_t tDK = tmem_base + C::kColDK;
      bool ok = steps > 0 && mbar_wait(kv_full, 0, abort_flag, a.status);
      for (int s = 0; s < steps && ok; ++s) {
        const int slot = s & 1;
        if (!(ok = mbar_wait(&q_full[slot], (s >> 1) & 1, abort_flag, a.status))) break;
        tc_fence_after();
        const uint32_t sQ = smem_u32(smem + C::kQ + slot * C::kQTile);
        const uint32_t sDO = smem_u32(smem + C::kDO + slot * C::kQTile);
        // S^T = K Q^T and dP^T = V dO^T: K-major operands, 16 elements (32 bytes)
        // per step inside a 128-byte swizzle row, then the next 64-column chunk.
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::kKVChunk + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::kQChunk + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(sK + okv, 16, 1024), sdesc_sw128(sQ + oq, 16, 1024), idesc_s,
                  kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::kKVChunk + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::kQChunk + (kk & 3) * 32;
          umma_ss(tDP, sdesc_sw128(sV + okv, 16, 1024), sdesc_sw128(sDO + oq, 16, 1024), idesc_s,
                  kk > 0);
        }
        umma_commit(s_full);
        if (!(ok = mbar_wait(p_ready, s & 1, abort_flag, a.status))) break;
        tc_fence_after();
        // dV += P^T dO (P^T from TMEM, two queries per column) and dK += dS^T Q:
        // dO and Q as N-contiguous B operands, 16 query rows (2048 bytes) per step.
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ts(tDV, tS + kk * 8, sdesc_sw128(sDO + kk * 2048, C::kQChunk, 1024), idesc_g,
                  (s > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ss(tDK, sdesc_sw128(sDS + (kk >> 2) * C::kKVChunk + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(sQ + kk * 2048, C::kQChunk, 1024), idesc_g,
                  (s > 0 || kk > 0) ? 1u : 0u);
        // dQ: both operands M/N-contiguous views of row-major 128-key tiles, 16 keys
        // (2048 bytes) per step.  K = 128: dQ^T = K^T dS^T; K = 64: dQ = dS K.
        if (s > 0) {
          if (!(ok = mbar_wait(dq_empty, (s - 1) & 1, abort_flag, a.status))) break;
          tc_fence_after();
        }
        const uint32_t qa = (D == 128) ? sK : sDS;
        const uint32_t qb = (D == 128) ? sDS : sK;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ss(tDQ, sdesc_sw128(qa + kk * 2048, C::kKVChunk, 1024),
                  sdesc_sw128(qb + kk * 2048, C::kKVChunk, 1024), idesc_q, kk > 0);
        umma_commit(dq_full);
        umma_commit(&q_empty[slot]);
      }
      // Every MMA issued above has completed once this barrier flips.
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, a.status);
    }
  } else if (warp < 4) {
    // ===================== P^T and dS^T, then the dK / dV epilogue ============
    const int row = warp * 32 + lane;  // key inside the block = TMEM lane
    const int j_loc = n0 + row;
    const bool key_ok = j_loc < k_len;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem_base + lane_addr + C::kColS;
    const uint32_t tDP = tmem_base + lane_addr + C::kColDP;
    uint8_t* ds_row = smem + C::kDS + row * 128;
    bool ok = true;
    for (int s = 0; s < steps && ok; ++s) {
      const int h = kvh * a.group + s / n_mblocks;
      const int m0 = m_first + (s % n_mblocks) * BM;
      const int slot = s & 1;
      float slope_log2 = 0.f;
      if constexpr (ALIBI) slope_log2 = exp2f(-8.0f * static_cast<float>(h + 1) / a.Hq) * kLog2e;
      // lse / D of this block were staged with the Q copy of the slot.
      if (!(ok = mbar_wait_warp(&q_full[slot], (s >> 1) & 1, abort_flag, a.status))) break;
      if (!(ok = mbar_wait_warp(s_full, s & 1, abort_flag, a.status))) break;
      tc_fence_after();
      const float* lse2 = s_lse + slot * BM;
      const float* dlt = s_delta + slot * BM;
#pragma unroll 1
      for (int c = 0; c < BM / 32; ++c) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + 32 * c, sr);
        tmem_ld32(tDP + 32 * c, dr);
        tmem_ld_wait(sr);
        tmem_ld_wait(dr);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qc = 32 * c + k + e;    // query column
            const int pos_i = m0 + qc + off;  // query position in key coordinates
            float x = fmaf(__uint_as_float(sr[k + e]), a.scale_log2, -lse2[qc]);
            if constexpr (ALIBI) x -= slope_log2 * fabsf(static_cast<float>(pos_i - j_loc));
            bool vis = key_ok;
            if constexpr (kCausal) vis = vis && j_loc <= pos_i;
            const float p = vis ? ex2(x) : 0.f;
            p2[e] = p;
            d2[e] = p * (__uint_as_float(dr[k + e]) - dlt[qc]);
          }
          pk[k / 2] = pack2<BF16>(p2[0], p2[1]);
          dk[k / 2] = pack2<BF16>(d2[0], d2[1]);
        }
        // P^T over S^T columns already read: queries 2c', 2c'+1 in column c'.
        tmem_st16(tS + 16 * c, pk);
        // dS^T row `row`, columns 32c..32c+31, in the 128-byte-swizzled layout the
        // MMA descriptors read: 16-byte piece u of a 64-column chunk sits at u ^ (row & 7).
        const int plane = (32 * c) >> 6;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int piece = (((32 * c) & 63) >> 3) + u;
          *reinterpret_cast<uint4*>(ds_row + plane * C::kKVChunk + ((piece ^ (row & 7)) << 4)) =
              make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_ready);
    }
    // ---- epilogue: dK (scaled) and dV of the valid keys ------------------------
    // The TMEM loads are warp-collective: every lane issues them, and only the
    // global stores depend on the lane's key.
    if (ok) ok = mbar_wait_warp(mma_done, 0, abort_flag, a.status);
    if (ok) {
      tc_fence_after();
      const long long grow = (static_cast<long long>(bidx) * a.N + k0 + j_loc) * a.Hkv + kvh;
      uint8_t* dk_row = static_cast<uint8_t*>(a.dk) + grow * D * 2;
      uint8_t* dv_row = static_cast<uint8_t*>(a.dv) + grow * D * 2;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t kr[32], vr[32];
        if (steps > 0) {
          tmem_ld32(tmem_base + lane_addr + C::kColDK + 32 * c, kr);
          tmem_ld32(tmem_base + lane_addr + C::kColDV + 32 * c, vr);
          tmem_ld_wait(kr);
          tmem_ld_wait(vr);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) kr[i] = vr[i] = 0u;
        }
        uint32_t pkk[16], pkv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pkk[i] = pack2<BF16>(__uint_as_float(kr[2 * i]) * a.scale,
                               __uint_as_float(kr[2 * i + 1]) * a.scale);
          pkv[i] = pack2<BF16>(__uint_as_float(vr[2 * i]), __uint_as_float(vr[2 * i + 1]));
        }
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            reinterpret_cast<uint4*>(dk_row + c * 64)[u] =
                make_uint4(pkk[4 * u], pkk[4 * u + 1], pkk[4 * u + 2], pkk[4 * u + 3]);
            reinterpret_cast<uint4*>(dv_row + c * 64)[u] =
                make_uint4(pkv[4 * u], pkv[4 * u + 1], pkv[4 * u + 2], pkv[4 * u + 3]);
          }
        }
      }
    }
  } else {
    // ===================== dQ drain (warps 4-7) ===============================
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // TMEM lane: a head dimension (K = 128) or a query (K = 64)
    const uint32_t t_addr = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + C::kColDQ;
    bool ok = true;
    for (int s = 0; s < steps && ok; ++s) {
      const int h = kvh * a.group + s / n_mblocks;
      const int m0 = m_first + (s % n_mblocks) * BM;
      if (!(ok = mbar_wait_warp(dq_full, s & 1, abort_flag, a.status))) break;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(t_addr, v0);
      tmem_ld32(t_addr + 32, v1);
      tmem_ld_wait(v0);
      tmem_ld_wait(v1);
      tc_fence_before();
      mbar_arrive(dq_empty);
      const long long row0 = (static_cast<long long>(bidx) * a.M + q0 + m0) * a.Hq + h;
      if constexpr (D == 128) {
        // lane = dimension `row`, columns = the block's 64 queries
        const int nq = min(64, q_len - m0);
        float* base = a.dq_acc + row0 * D + row;
        const long long qstride = static_cast<long long>(a.Hq) * D;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < nq) red_add(base + k * qstride, __uint_as_float(v0[k]) * a.scale);
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (32 + k < nq) red_add(base + (32 + k) * qstride, __uint_as_float(v1[k]) * a.scale);
      } else {
        // lane = query m0 + row, columns = its 64 dimensions
        if (m0 + row < q_len) {
          float* dst = a.dq_acc + (row0 + static_cast<long long>(row) * a.Hq) * D;
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            red_add4(dst + k, __uint_as_float(v0[k]) * a.scale,
                     __uint_as_float(v0[k + 1]) * a.scale, __uint_as_float(v0[k + 2]) * a.scale,
                     __uint_as_float(v0[k + 3]) * a.scale);
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            red_add4(dst + 32 + k, __uint_as_float(v1[k]) * a.scale,
                     __uint_as_float(v1[k + 1]) * a.scale, __uint_as_float(v1[k + 2]) * a.scale,
                     __uint_as_float(v1[k + 3]) * a.scale);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int D, bool BF16, int MASK, bool ALIBI>
cudaError_t launch_main(const BwdLaunch& L, cudaStream_t stream) {
  auto kern = bwd_kernel<D, BF16, MASK, ALIBI>;
  const int smem = BwdCfg<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const BwdArgs& a = L.args;
  dim3 grid(a.num_kblocks, a.Hkv, a.num_units);
  kern<<<grid, kThreads, smem, stream>>>(L.tmQ, L.tmK, L.tmV, L.tmDO, a);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_all(const BwdLaunch& L, cudaStream_t stream) {
  const BwdArgs& a = L.args;
  const long long rows = static_cast<long long>(a.B) * a.M * a.Hq;
  if (rows <= 0) return cudaSuccess;
  bwd_prep_kernel<D, BF16><<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.num_kblocks > 0 && a.N > 0) {
    switch (L.mask * 2 + (L.alibi ? 1 : 0)) {
      case 0: e = launch_main<D, BF16, 0, false>(L, stream); break;
      case 1: e = launch_main<D, BF16, 0, true>(L, stream); break;
      case 2: e = launch_main<D, BF16, 1, false>(L, stream); break;
      case 3: e = launch_main<D, BF16, 1, true>(L, stream); break;
      case 4: e = launch_main<D, BF16, 2, false>(L, stream); break;
      case 5: e = launch_main<D, BF16, 2, true>(L, stream); break;
      case 6: e = launch_main<D, BF16, 3, false>(L, stream); break;
      case 7: e = launch_main<D, BF16, 3, true>(L, stream); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  const long long pairs = rows * D / 2;
  const long long blocks = std::min((pairs + 255) / 256, 148LL * 16);
  bwd_dq_out_kernel<D, BF16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

int bwd_query_block(int head_dim) { return head_dim == 128 ? BwdCfg<128>::BM : BwdCfg<64>::BM; }

cudaError_t launch_bwd(const BwdLaunch& L, cudaStream_t stream) {
  if (L.head_dim == 64)
    return L.bf16 ? launch_all<64, true>(L, stream) : launch_all<64, false>(L, stream);
  if (L.head_dim == 128)
    return L.bf16 ? launch_all<128, true>(L, stream) : launch_all<128, false>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mea
