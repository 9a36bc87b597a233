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
//   P^T, dS^T from S^T, dP^T, lse_i, D_i               (256 threads, two per key)
//     P^T (16-bit) to its own TMEM columns, dS^T to shared memory (two buffers)
//   dV  += P^T dO_i   (A = P^T from TMEM)              dK += dS^T Q_i
//   dQ_i = dS_i K  (K = 64)  or  dQ_i^T = K^T dS_i^T (K = 128): both M = 128, N = 64
//   dQ_i is drained by four warps: scaled, staged in a shared-memory buffer of its
//   own and added to the fp32 accumulator by TMA tensor reductions (one per 32
//   columns).
// The S^T / dP^T columns are released as soon as the P/dS threads have read
// them, so the MMA thread issues the next block's S^T, dP^T before this block's
// dV, dK, dQ and the P/dS arithmetic of one block overlaps the MMAs of its
// neighbours.  dS^T of block i goes to buffer i % 2, last read by block i-2's
// MMAs, which completed before block i's S^T did (issue order); P^T of block i
// is stored once block i-1's MMAs are done.
//
// CTA (448 threads): warps 0-7 P/dS and the dK/dV epilogue (warps w and w+4
// share TMEM lane quarter w, each taking half of the query columns, read 16 at a
// time), warps 8-11 the dQ drain, warp 12 allocates TMEM and issues every MMA,
// warp 13 loads (one thread issues the TMA copies; the warp stages lse and D).
// The MMA warp runs its issuing loop warp-wide; elect.sync picks the lane that
// issues each MMA and commit.
#include <math.h>

#include <algorithm>

#include <type_traits>

#include "mea_internal.h"
#include "sm100.cuh"

namespace mea {
namespace {

constexpr int kBN = kBwdBlock;  // keys per CTA (= TMEM lanes)
constexpr int kPdsWarps = 8;  // P/dS warps: two per TMEM lane quarter (a column half each)
constexpr int kThreads = (kPdsWarps + 6) * 32;
constexpr int kDrainWarp = kPdsWarps;  // four drain warps
constexpr int kMmaWarp = kPdsWarps + 4;
constexpr int kLoadWarp = kPdsWarps + 5;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Wait until every bulk async-group of this thread but the most recent one has
// finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}



// Pipeline timeline for performance work: built only with -DMEA_TRACE, it
// records clock64() at pipeline events of the first kBwdTraceCtas CTAs.
// Slots per CTA: step s (< 64), event e (< 32) -> s*32 + e; CTA-level events at
// 2048 + e.
#ifdef MEA_TRACE
constexpr int kBwdTraceCtas = 4;
constexpr int kBwdTraceSlots = 2048 + 32;
__device__ long long g_bwd_trace[kBwdTraceCtas * kBwdTraceSlots];
#define BWD_TRACE(s, e)                                                                   \
  do {                                                                                    \
    const int cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);      \
    const int slot_ = (s) < 64 ? (s) * 32 + (e) : -1;                                     \
    if (cta_ < kBwdTraceCtas && slot_ >= 0) g_bwd_trace[cta_ * kBwdTraceSlots + slot_] = clock64(); \
  } while (0)
#define BWD_TRACE_CTA(e)                                                                  \
  do {                                                                                    \
    const int cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);      \
    if (cta_ < kBwdTraceCtas) g_bwd_trace[cta_ * kBwdTraceSlots + 2048 + (e)] = clock64(); \
  } while (0)
#else
#define BWD_TRACE(s, e) \
  do {                  \
  } while (0)
#define BWD_TRACE_CTA(e) \
  do {                   \
  } while (0)
#endif

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
  // Q / dO stages: three (two steps of look-ahead for the loads).
  static constexpr int kStages = 3;
  static constexpr int kStage = 2 * kQTile;           // Q then dO
  // dQ staging, in boxes of kDQRows rows x 32 fp32 (128 B a row).  K = 128: the
  // D/32 boxes of one half step (32 queries) at a time, in two buffers, so one
  // half is staged while the other's reductions read it; K = 64 (BM = 128): one
  // 32-dimension box of the step at a time, which leaves room for the third Q / dO
  // stage.
  static constexpr int kDQRows = (D == 128) ? 32 : BM;
  static constexpr int kDQSBox = kDQRows * 128;
  static constexpr int kDQSBoxes = (D == 128) ? 2 * (D / 32) : 1;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int kK = 0;
  static constexpr int kV = kKVTile;
  static constexpr int kQD = 2 * kKVTile;              // stage i: Q at kQD + i*kStage, dO after it
  static constexpr int kDS = kQD + kStages * kStage;   // two buffers (step parity)
  static constexpr int kDQS = kDS + 2 * kDSTile;       // dQ of one step, fp32, for the reductions
  static constexpr int kLse = kDQS + kDQSBoxes * kDQSBox;  // [stage][BM] -lse * log2(e) (-inf: no weight)
  static constexpr int kDelta = kLse + kStages * BM * 4;  // [stage][BM] -D
  static constexpr int kBar = kDelta + kStages * BM * 4;
  static constexpr int kNumBars = 14;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;
  static_assert(kBytes <= 227 * 1024, "shared memory");
  // tensor memory columns (every region starts on a multiple of 64):
  //   K = 64:  S^T 0 | dP^T 128 | P^T 256 (64) | dQ 320 | dV 384 | dK 448
  //   K = 128: S^T 0 | dP^T 64 | dQ 128 | dV 192 | dK 320 | P^T 448 (32)
  static constexpr uint32_t kColS = 0, kColDP = BM;
  static constexpr uint32_t kColP = (D == 64) ? 256 : 448;
  static constexpr uint32_t kColDQ = (D == 64) ? 320 : 128;
  static constexpr uint32_t kColDV = (D == 64) ? 384 : 192;
  static constexpr uint32_t kColDK = (D == 64) ? 448 : 320;
  static_assert(kColDK + D <= kTmemCols && kColP + BM / 2 <= kTmemCols, "tensor memory layout");
};

// D = <dout, out> per (row, query head), and the row's dq accumulator zeroed.
// A row is K / 8 lanes of 16-byte loads (8 at K = 64, 16 at K = 128), so a warp
// covers 4 or 2 rows with fully used 16-byte accesses.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  constexpr int kLanes = D / 8;  // lanes per row, 8 elements each
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / kLanes;
  const int part = static_cast<int>(t % kLanes);
  const long long rows = static_cast<long long>(a.B) * a.M * a.Hq;
  const bool live = row < rows;
  float s = 0.f;
  if (live) {
    const uint4 o = reinterpret_cast<const uint4*>(a.out)[row * kLanes + part];
    const uint4 g = reinterpret_cast<const uint4*>(a.dout)[row * kLanes + part];
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      s = fmaf(to_f<BF16>(static_cast<uint16_t>(ow[w] & 0xffffu)),
               to_f<BF16>(static_cast<uint16_t>(gw[w] & 0xffffu)), s);
      s = fmaf(to_f<BF16>(static_cast<uint16_t>(ow[w] >> 16)),
               to_f<BF16>(static_cast<uint16_t>(gw[w] >> 16)), s);
    }
    float4* acc = reinterpret_cast<float4*>(a.dq_acc + row * D + part * 8);
    acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (live && part == 0) {
    const long long b = row / (static_cast<long long>(a.M) * a.Hq);
    const long long i = (row / a.Hq) % a.M;
    const long long h = row % a.Hq;
    a.delta[(b * a.Hq + h) * a.M + i] = s;
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_dq_out_kernel(const BwdArgs a) {
  const long long n = static_cast<long long>(a.B) * a.M * a.Hq * D / 4;  // 4 elements each
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(a.dq_acc)[e];
    reinterpret_cast<uint2*>(a.dq)[e] = make_uint2(pack2<BF16>(v.x, v.y), pack2<BF16>(v.z, v.w));
  }
}

template <int D, bool BF16, int MASK, bool ALIBI>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM;
  constexpr bool kCausal = (MASK == 1 || MASK == 3);
  constexpr bool kPacked = (MASK >= 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  constexpr int NS = C::kStages;
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;        // [NS] Q, dO (+ lse, D) of a step landed
  uint64_t* q_empty = bars + 1 + NS;  // [NS] the stage is free again (its MMAs completed)
  uint64_t* s_full = bars + 1 + 2 * NS;   // S^T, dP^T of the step are in TMEM
  uint64_t* s_free = s_full + 1;      // S^T, dP^T read out of TMEM (256 arrivals)
  uint64_t* p_ready = s_full + 2;     // P^T in TMEM and dS^T in shared memory (256 arrivals)
  uint64_t* p_done = s_full + 3;      // the step's dV, dK, dQ MMAs completed
  uint64_t* dq_full = s_full + 4;     // dQ of the step is in TMEM
  uint64_t* dq_empty = s_full + 5;    // dQ read out of TMEM (128 arrivals)
  uint64_t* mma_done = s_full + 6;
  float* s_lse = reinterpret_cast<float*>(smem + C::kLse);
  float* s_delta = reinterpret_cast<float*>(smem + C::kDelta);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA -> (key block, kv head, batch or sequence).  Under a causal mask a key
  // block's work falls with its index (block 0 sees every query row, the last
  // block only the last rows), so the key block varies slowest and the heaviest
  // CTAs of the launch start first; otherwise it varies fastest, so the CTAs of
  // one (kv head, batch) run together and share their Q / dO reads in L2.
  int nb = blockIdx.x, kvh = blockIdx.y, unit = blockIdx.z;
  if constexpr (MASK == 1 || MASK == 3) {
    const int l = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int per = gridDim.y * gridDim.z;
    nb = l / per;
    kvh = (l - nb * per) % gridDim.y;
    unit = (l - nb * per) / gridDim.y;
  }

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
    for (int s = 0; s < NS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kPdsWarps);  // one arrival per P/dS warp
    mbar_init(p_ready, kPdsWarps);
    mbar_init(p_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 4);  // one arrival per dQ drain warp
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
  if (threadIdx.x == 0) BWD_TRACE_CTA(0);

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
      const int slot = s % NS;
      // -lse (log2 units) and -D of the block's rows, fetched before waiting for
      // the stage; -inf marks a row that takes no weight (past the sequence, or
      // no visible key in the forward).
      float l2[BM / 32], dl[BM / 32];
#pragma unroll
      for (int u = 0; u < BM / 32; ++u) {
        const int i = m0 + u * 32 + lane;
        l2[u] = neg_inf();
        dl[u] = 0.f;
        if (i < q_len) {
          const long long li = (static_cast<long long>(bidx) * a.Hq + h) * a.M + q0 + i;
          l2[u] = a.lse[li];
          dl[u] = a.delta[li];
        }
      }
      if (!(ok = mbar_wait_warp(&q_empty[slot], ((s / NS) & 1) ^ 1, abort_flag, a.status))) break;
      if (lane == 0) {
        BWD_TRACE(s, 24);
        mbar_expect_tx(&q_full[slot], C::kStage);
        uint8_t* st = smem + C::kQD + slot * C::kStage;
        for (int c = 0; c < C::kChunksD; ++c) {
          tma_load_4d(st + c * C::kQChunk, &tmQ, &q_full[slot], c * 64, h, q0 + m0, bidx);
          tma_load_4d(st + C::kQTile + c * C::kQChunk, &tmDO, &q_full[slot], c * 64, h, q0 + m0,
                      bidx);
        }
      }
#pragma unroll
      for (int u = 0; u < BM / 32; ++u) {
        s_lse[slot * BM + u * 32 + lane] = l2[u] == neg_inf() ? neg_inf() : -l2[u] * kLog2e;
        s_delta[slot * BM + u * 32 + lane] = -dl[u];
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&q_full[slot]);
        BWD_TRACE(s, 25);
      }
      issued = s + 1;
    }
    // Let every copy this warp started land before the CTA can exit.
    if (lane == 0 && steps > 0) {
      mbar_wait_drain(kv_full, 0, a.status);
      for (int s = max(0, issued - NS); s < issued; ++s)
        mbar_wait_drain(&q_full[s % NS], (s / NS) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ===================== MMA issue (one warp) ==============================
    // The whole warp runs the loop (all values warp-uniform); elect.sync picks the
    // lane that issues each MMA and commit.
    {
      constexpr uint32_t idesc_s = idesc_f16_ab(BF16, kBN, BM, false, false);
      constexpr uint32_t idesc_g = idesc_f16_ab(BF16, kBN, D, false, true);
      constexpr uint32_t idesc_q = idesc_f16_ab(BF16, kBN, 64, true, true);
      const uint32_t sK = smem_u32(smem + C::kK), sV = smem_u32(smem + C::kV);
      const uint32_t sDS0 = smem_u32(smem + C::kDS);
      const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP;
      const uint32_t tDQ = tmem_base + C::kColDQ, tDV = tmem_base + C::kColDV;
      const uint32_t tDK = tmem_base + C::kColDK;
      const uint32_t tP = tmem_base + C::kColP;
      // S^T = K Q^T and dP^T = V dO^T of step `st`: K-major operands, 16 elements
      // (32 bytes) per step inside a 128-byte swizzle row, then the next chunk.
      auto issue_s = [&](int st) {
        const uint32_t sQ = smem_u32(smem + C::kQD + (st % NS) * C::kStage);
        const uint32_t sDO = sQ + C::kQTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::kKVChunk + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::kQChunk + (kk & 3) * 32;
          umma_ss_warp(tS, sdesc_sw128(sK + okv, 16, 1024), sdesc_sw128(sQ + oq, 16, 1024), idesc_s,
                  kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::kKVChunk + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::kQChunk + (kk & 3) * 32;
          umma_ss_warp(tDP, sdesc_sw128(sV + okv, 16, 1024), sdesc_sw128(sDO + oq, 16, 1024), idesc_s,
                  kk > 0);
        }
        umma_commit_warp(s_full);
      };
      bool ok = steps > 0 && mbar_wait_warp(kv_full, 0, abort_flag, a.status) &&
                mbar_wait_warp(&q_full[0], 0, abort_flag, a.status);
      if (ok) {
        BWD_TRACE_CTA(1);
        tc_fence_after();
        issue_s(0);
      }
      for (int s = 0; s < steps && ok; ++s) {
        const int slot = s % NS;
        // The next block's scores go first: they only need its Q / dO and the
        // S^T / dP^T columns, which the P/dS threads have read out.
        if (s + 1 < steps) {
          if (!(ok = mbar_wait_warp(&q_full[(s + 1) % NS], ((s + 1) / NS) & 1, abort_flag, a.status)))
            break;
          BWD_TRACE(s, 0);
          if (!(ok = mbar_wait_warp(s_free, s & 1, abort_flag, a.status))) break;
          BWD_TRACE(s, 1);
          tc_fence_after();
          issue_s(s + 1);
          BWD_TRACE(s, 2);
        }
        if (!(ok = mbar_wait_warp(p_ready, s & 1, abort_flag, a.status))) break;
        BWD_TRACE(s, 3);
        tc_fence_after();
        const uint32_t sQ = smem_u32(smem + C::kQD + slot * C::kStage);
        const uint32_t sDO = sQ + C::kQTile;
        const uint32_t sDS = sDS0 + (s & 1) * C::kDSTile;
        // dV += P^T dO (P^T from TMEM, two queries per column) and dK += dS^T Q:
        // dO and Q as N-contiguous B operands, 16 query rows (2048 bytes) per step.
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ts_warp(tDV, tP + kk * 8, sdesc_sw128(sDO + kk * 2048, C::kQChunk, 1024), idesc_g,
                  (s > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ss_warp(tDK, sdesc_sw128(sDS + (kk >> 2) * C::kKVChunk + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(sQ + kk * 2048, C::kQChunk, 1024), idesc_g,
                  (s > 0 || kk > 0) ? 1u : 0u);
        // No later MMA reads this step's Q / dO stage: the loader may refill it
        // once these have completed.
        umma_commit_warp(&q_empty[slot]);
        // dQ: both operands M/N-contiguous views of row-major 128-key tiles, 16 keys
        // (2048 bytes) per step.  K = 128: dQ^T = K^T dS^T; K = 64: dQ = dS K.
        BWD_TRACE(s, 4);
        if (s > 0) {
          if (!(ok = mbar_wait_warp(dq_empty, (s - 1) & 1, abort_flag, a.status))) break;
          tc_fence_after();
        }
        BWD_TRACE(s, 5);
        const uint32_t qa = (D == 128) ? sK : sDS;
        const uint32_t qb = (D == 128) ? sDS : sK;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ss_warp(tDQ, sdesc_sw128(qa + kk * 2048, C::kKVChunk, 1024),
                  sdesc_sw128(qb + kk * 2048, C::kKVChunk, 1024), idesc_q, kk > 0);
        umma_commit_warp(dq_full);
        umma_commit_warp(p_done);
        BWD_TRACE(s, 6);
      }
      // Every MMA issued above has completed once this barrier flips.
      umma_commit_warp(mma_done);
      mbar_wait_drain(mma_done, 0, a.status);
    }
  } else if (warp < kPdsWarps) {
    // ===================== P^T and dS^T, then the dK / dV epilogue ============
    constexpr int kParts = kPdsWarps / 4;  // warps sharing a TMEM lane quarter
    constexpr int kCols = BM / kParts;     // query columns per thread (64 at K = 64, 32 at 128)
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;  // key inside the block = TMEM lane
    const int c0 = part * kCols;          // this thread's first query column
    const int j_loc = n0 + row;
    const bool key_ok = j_loc < k_len;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_addr + C::kColS + c0;
    const uint32_t tDP = tmem_base + lane_addr + C::kColDP + c0;
    const uint32_t tP = tmem_base + lane_addr + C::kColP + c0 / 2;
    uint8_t* ds_row = smem + C::kDS + row * 128;
    const f2 scale2 = {a.scale_log2, a.scale_log2};
    const f2 zero2 = {0.f, 0.f};
    bool ok = true;
    for (int s = 0; s < steps && ok; ++s) {
      const int h = kvh * a.group + s / n_mblocks;
      const int m0 = m_first + (s % n_mblocks) * BM;
      const int slot = s % NS;
      float slope_log2 = 0.f;
      if constexpr (ALIBI) slope_log2 = exp2f(-8.0f * static_cast<float>(h + 1) / a.Hq) * kLog2e;
      const bool tracer = warp == 0 && lane == 0;
      if (tracer) BWD_TRACE(s, 13);
      // -lse / -D of this block were staged with the Q copy of the stage.
      if (!(ok = mbar_wait_warp(&q_full[slot], (s / NS) & 1, abort_flag, a.status))) break;
      if (tracer) BWD_TRACE(s, 14);
      if (!(ok = mbar_wait_warp(s_full, s & 1, abort_flag, a.status))) break;
      if (tracer) BWD_TRACE(s, 8);
      tc_fence_after();
      // Per-element masks only where the tile reaches past the keys or past the
      // diagonal for this thread's queries.
      const bool full =
          n0 + kBN <= k_len && (!kCausal || m0 + c0 + off >= n0 + kBN - 1);
      const float* nl = s_lse + slot * BM + c0;
      const float* nd = s_delta + slot * BM + c0;
      uint8_t* ds_buf = ds_row + (s & 1) * C::kDSTile;
      uint32_t pk[kCols / 2];
      // K = 128: instantiated for blocks with and without per-element masks, so
      // the unmasked copy carries no mask arithmetic (`full` depends on the warp
      // only, through c0, as the warp-collective TMEM loads inside require).
      // K = 64: one copy with a run-time test (two copies spill there).
      auto p_ds = [&](auto msk) {
        // kChunk columns at a time: read S^T, dP^T out of TMEM (releasing them after
        // the last chunk), then P = 2^(s*scale*log2e - lse*log2e) and dS = P (dP - D).
        constexpr int kChunk = 16;
#pragma unroll
        for (int c = 0; c < kCols / kChunk; ++c) {
          uint32_t sr[kChunk], dr[kChunk], dk[kChunk / 2];
          tmem_ld2x16_wait(tS + kChunk * c, tDP + kChunk * c, sr, dr);
          if (c == kCols / kChunk - 1) {
            tc_fence_before();
            mbar_arrive_warp(s_free);  // the next block's S^T / dP^T may be written now
            if (tracer) BWD_TRACE(s, 9);
          }
#pragma unroll
          for (int e = 0; e < kChunk; e += 2) {
            const int k = kChunk * c + e;
            const float2 l = *reinterpret_cast<const float2*>(nl + k);
            const float2 dd = *reinterpret_cast<const float2*>(nd + k);
            f2 x = fma2(f2{__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])}, scale2,
                        f2{l.x, l.y});
            [[maybe_unused]] const int pos = m0 + c0 + k + off;  // query position of column k, key coordinates
            if constexpr (ALIBI) {
              x.x -= slope_log2 * fabsf(static_cast<float>(pos - j_loc));
              x.y -= slope_log2 * fabsf(static_cast<float>(pos + 1 - j_loc));
            }
            f2 p = {ex2(x.x), ex2(x.y)};
            if (flag_on(msk)) {
              bool v0 = key_ok, v1 = key_ok;
              if constexpr (kCausal) {
                v0 = v0 && j_loc <= pos;
                v1 = v1 && j_loc <= pos + 1;
              }
              if (!v0) p.x = 0.f;
              if (!v1) p.y = 0.f;
            }
            const f2 t = add2(f2{__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])},
                              f2{dd.x, dd.y});
            const f2 ds = fma2(p, t, zero2);
            pk[k / 2] = pack2<BF16>(p.x, p.y);
            dk[e / 2] = pack2<BF16>(ds.x, ds.y);
          }
          // dS^T row `row`, columns c0 + kChunk c .. + kChunk - 1, in the 128-byte-swizzled
          // layout the MMA descriptors read: 16-byte piece u of a 64-column chunk sits at
          // u ^ (row & 7).
          const int col = c0 + kChunk * c;
          const int plane = col >> 6;
#pragma unroll
          for (int u = 0; u < kChunk / 8; ++u) {
            const int piece = ((col & 63) >> 3) + u;
            *reinterpret_cast<uint4*>(ds_buf + plane * C::kKVChunk + ((piece ^ (row & 7)) << 4)) =
                make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
          }
        }
      };
      if constexpr (D == 128) {
        if (full) p_ds(std::false_type{});
        else p_ds(std::true_type{});
      } else {
        p_ds(!full);
      }
      if (tracer) BWD_TRACE(s, 10);
      // The previous block's dV MMAs still read P^T (queries 2c, 2c+1 in column c).
      if (s > 0 && !(ok = mbar_wait_warp(p_done, (s - 1) & 1, abort_flag, a.status))) break;
      if (tracer) BWD_TRACE(s, 11);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kCols / 32; ++c) tmem_st16(tP + 16 * c, pk + 16 * c);
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive_warp(p_ready);
      if (tracer) BWD_TRACE(s, 12);
    }
    // ---- epilogue: dK (scaled) and dV of the valid keys, D / kParts columns each --
    // The TMEM loads are warp-collective: every lane issues them, and only the
    // global stores depend on the lane's key.
    if (ok) ok = mbar_wait_warp(mma_done, 0, abort_flag, a.status);
    if (warp == 0 && lane == 0) BWD_TRACE_CTA(2);
    if (ok) {
      tc_fence_after();
      const int dc0 = part * (D / kParts);
      const long long grow = (static_cast<long long>(bidx) * a.N + k0 + j_loc) * a.Hkv + kvh;
      uint8_t* dk_row = static_cast<uint8_t*>(a.dk) + (grow * D + dc0) * 2;
      uint8_t* dv_row = static_cast<uint8_t*>(a.dv) + (grow * D + dc0) * 2;
#pragma unroll 1
      for (int c = 0; c < D / kParts / 16; ++c) {
        uint32_t kr[16], vr[16];
        if (steps > 0) {
          tmem_ld2x16_wait(tmem_base + lane_addr + C::kColDK + dc0 + 16 * c,
                           tmem_base + lane_addr + C::kColDV + dc0 + 16 * c, kr, vr);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) kr[i] = vr[i] = 0u;
        }
        uint32_t pkk[8], pkv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pkk[i] = pack2<BF16>(__uint_as_float(kr[2 * i]) * a.scale,
                               __uint_as_float(kr[2 * i + 1]) * a.scale);
          pkv[i] = pack2<BF16>(__uint_as_float(vr[2 * i]), __uint_as_float(vr[2 * i + 1]));
        }
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            reinterpret_cast<uint4*>(dk_row + c * 32)[u] =
                make_uint4(pkk[4 * u], pkk[4 * u + 1], pkk[4 * u + 2], pkk[4 * u + 3]);
            reinterpret_cast<uint4*>(dv_row + c * 32)[u] =
                make_uint4(pkv[4 * u], pkv[4 * u + 1], pkv[4 * u + 2], pkv[4 * u + 3]);
          }
        }
      }
    }
  } else {
    // ===================== dQ drain (warps 16-19) =============================
    // dQ of a step goes TMEM -> registers (scaled) -> a 128-byte-swizzled staging
    // tile in shared memory, whose 32-column boxes are added to the fp32
    // accumulator by TMA reductions issued by one thread.
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // TMEM lane: a head dimension (K = 128) or a query (K = 64)
    const bool leader = (warp == kDrainWarp && lane == 0);
    const uint32_t t_addr = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + C::kColDQ;
    bool ok = true;
    for (int s = 0; s < steps && ok; ++s) {
      const int h = kvh * a.group + s / n_mblocks;
      const int m0 = m_first + (s % n_mblocks) * BM;
      if (!(ok = mbar_wait_warp(dq_full, s & 1, abort_flag, a.status))) break;
      if (leader) BWD_TRACE(s, 16);
      tc_fence_after();
      // Stage dQ in the staging buffer, once the previous reductions have read it
      // (the leader waits for them, then joins barrier 2).
      uint8_t* stage = smem + C::kDQS;
      // K = 64: the one staged box (dims 32b .. 32b + 31) into the accumulator.
      auto reduce_box = [&](int b) {
        fence_async_smem();
        named_sync(1, 128);
        if (leader) {
          BWD_TRACE(s, 17);
          tma_reduce_add_4d(&tmDQ, stage, 32 * b, h, q0 + m0, bidx);
          bulk_commit();
          bulk_wait_read();  // the staging buffer may be written again
        }
      };
      if constexpr (D == 64) {
        // Both 32-column halves come out of TMEM first, so dQ's columns are handed
        // back before the one-box-at-a-time staging and reductions.
        uint32_t v0[32], v1[32];
        tmem_ld32(t_addr, v0);
        tmem_ld32(t_addr + 32, v1);
        tmem_ld_wait(v0);
        tmem_ld_wait(v1);
        tc_fence_before();
        mbar_arrive_warp(dq_empty);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t(&v)[32] = half ? v1 : v0;
          if (s > 0 || half > 0) named_sync(2, 128);
          // lane = query m0 + row, columns = dims 32 half .. +31 = box `half`:
          // 16-byte piece u at u ^ (row & 7).
          const float sc = (m0 + row < q_len) ? a.scale : 0.f;
          uint8_t* line = stage + row * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4*>(line + ((u ^ (row & 7)) << 4)) =
                make_float4(__uint_as_float(v[4 * u]) * sc, __uint_as_float(v[4 * u + 1]) * sc,
                            __uint_as_float(v[4 * u + 2]) * sc, __uint_as_float(v[4 * u + 3]) * sc);
          reduce_box(half);
        }
      } else {
        // Half h (queries 32h .. 32h + 31) goes to buffer h; before a buffer is
        // written again the leader has seen the reductions that read it two
        // halves earlier complete (it keeps at most one group in flight).
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {  // 32 TMEM columns at a time
          if (s > 0 || half > 0) named_sync(2, 128);
          uint32_t v[32];
          tmem_ld32(t_addr + 32 * half, v);
          tmem_ld_wait(v);
          if (half == 1) {
            tc_fence_before();
            mbar_arrive_warp(dq_empty);
          }
          // lane = dimension `row`, columns = queries 32 half .. +31: element
          // (query k, dim row) of box row/32 at row k, byte 4 (row % 32), swizzled.
          uint8_t* buf = stage + half * (C::kDQSBoxes / 2) * C::kDQSBox;
          uint8_t* box = buf + (row >> 5) * C::kDQSBox;
          const int piece = (row & 31) >> 2, word = (row & 3) * 4;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int q = 32 * half + k;
            const float x = (m0 + q < q_len) ? __uint_as_float(v[k]) * a.scale : 0.f;
            *reinterpret_cast<float*>(box + k * 128 + ((piece ^ (k & 7)) << 4) + word) = x;
          }
          fence_async_smem();
          named_sync(1, 128);
          if (leader) {
            BWD_TRACE(s, 17);
#pragma unroll
            for (int b = 0; b < D / 32; ++b)
              tma_reduce_add_4d(&tmDQ, buf + b * C::kDQSBox, 32 * b, h, q0 + m0 + 32 * half, bidx);
            bulk_commit();
            bulk_wait_read_all_but_one();  // the other buffer may be written again
          }
        }
      }
    }
    if (leader) bulk_wait_all();
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
  constexpr auto kern = bwd_kernel<D, BF16, MASK, ALIBI>;
  const int smem = BwdCfg<D>::kBytes;
  cudaError_t e = set_smem_once<kern>(smem);
  if (e != cudaSuccess) return e;
  const BwdArgs& a = L.args;
  dim3 grid(a.num_kblocks, a.Hkv, a.num_units);
  kern<<<grid, kThreads, smem, stream>>>(L.tmQ, L.tmK, L.tmV, L.tmDO, L.tmDQ, a);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_all(const BwdLaunch& L, cudaStream_t stream, int stages) {
  const BwdArgs& a = L.args;
  const long long rows = static_cast<long long>(a.B) * a.M * a.Hq;
  if (rows <= 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (stages & 1) {
    bwd_prep_kernel<D, BF16>
      <<<static_cast<unsigned>((rows * (D / 8) + 255) / 256), 256, 0, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if ((stages & 2) && a.num_kblocks > 0 && a.N > 0) {
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
  if (!(stages & 4)) return cudaSuccess;
  const long long quads = rows * D / 4;
  const long long blocks = std::min((quads + 255) / 256, 148LL * 16);
  bwd_dq_out_kernel<D, BF16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

#ifdef MEA_TRACE
// Copies the recorded backward timeline (kBwdTraceCtas x kBwdTraceSlots clock64 values).
extern "C" int mea_bwd_trace_read(long long* host, int n) {
  if (n > kBwdTraceCtas * kBwdTraceSlots) n = kBwdTraceCtas * kBwdTraceSlots;
  return cudaMemcpyFromSymbol(host, g_bwd_trace, n * sizeof(long long)) == cudaSuccess ? n : -1;
}
#endif

int bwd_query_block(int head_dim) { return head_dim == 128 ? BwdCfg<128>::BM : BwdCfg<64>::BM; }

int bwd_dq_box_rows(int head_dim) {
  return head_dim == 128 ? BwdCfg<128>::kDQRows : BwdCfg<64>::kDQRows;
}

cudaError_t launch_bwd(const BwdLaunch& L, cudaStream_t stream, int stages) {
  if (L.head_dim == 64)
    return L.bf16 ? launch_all<64, true>(L, stream, stages)
                  : launch_all<64, false>(L, stream, stages);
  if (L.head_dim == 128)
    return L.bf16 ? launch_all<128, true>(L, stream, stages)
                  : launch_all<128, false>(L, stream, stages);
  return cudaErrorInvalidValue;
}

}  // namespace mea
