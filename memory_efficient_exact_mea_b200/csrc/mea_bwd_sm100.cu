// mea_bwd_sm100.cu -- attention backward: dq, dk, dv.
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
//   bwd_main     one CTA per (64-key block, kv head, batch or sequence): keeps dK
//                and dV of its keys in registers, loops over the query heads of
//                the group and the 64-row query blocks that can see its keys,
//                recomputes P, forms dP and dS, accumulates dV += P^T dO and
//                dK += dS^T Q, and adds dS K into dq with fp32 atomics;
//   bwd_dq_out   dq accumulator -> fp16/bf16.
// The contractions use mma.sync m16n8k16 with fp32 accumulation (8 warps: for
// the 64x64 score tiles each warp owns 16 rows x 32 keys, for the 64 x K
// gradient tiles 16 rows (or keys) x K/2 dims).  With bf16, P and dS enter the
// contractions as hi + lo pairs, as in the forward.
#include <math.h>

#include <algorithm>

#include "mea_internal.h"
#include "sm100.cuh"

namespace mea {
namespace {

constexpr int kBT = kBwdBlock;
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <bool BF16>
__device__ __forceinline__ float to_f(uint16_t x) {
  if constexpr (BF16) return __uint_as_float(static_cast<uint32_t>(x) << 16);
  else return __half2float(__ushort_as_half(x));
}

// Byte offset of 16-byte chunk `c` of row `r` in a shared tile whose rows are
// `row_bytes` long: chunks are XOR-swizzled within each group of eight so that
// eight consecutive rows at one chunk hit eight different bank groups.
__device__ __forceinline__ uint32_t sw(int r, int c, int row_bytes) {
  return r * row_bytes + (((c & ~7) | ((c ^ r) & 7)) << 4);
}

template <int D, bool BF16>
struct BSmem {
  static constexpr int kRow = D * 2;              // bytes per row of a K-wide tile
  static constexpr int kTile = kBT * kRow;
  static constexpr int kK = 0, kV = kTile, kQ = 2 * kTile, kDO = 3 * kTile;
  static constexpr int kPT = kBT * kBT * 2;       // one 64x64 16-bit tile
  static constexpr int kP = 4 * kTile;            // P_hi, dS_hi, then (bf16) P_lo, dS_lo
  static constexpr int kDS = kP + kPT;
  static constexpr int kPlo = kP + 2 * kPT, kDSlo = kP + 3 * kPT;
  static constexpr int kLse = kP + (BF16 ? 4 : 2) * kPT;
  static constexpr int kDelta = kLse + kBT * 4;
  static constexpr int kBytes = kDelta + kBT * 4;
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

// Copies rows [r0, r0 + 64) of a [rows, heads, D] 16-bit tensor (head h, row
// stride `row_stride` elements) into a swizzled shared tile; rows at or past
// `r_end` are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const uint16_t* base, long long r0,
                                          long long r_end, long long row_stride, int h) {
  constexpr int kChunks = D / 8;
  for (int e = threadIdx.x; e < kBT * kChunks; e += kThreads) {
    const int r = e / kChunks, c = e % kChunks;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    const long long gr = r0 + r;
    if (gr < r_end)
      v = *reinterpret_cast<const uint4*>(base + gr * row_stride + static_cast<long long>(h) * D +
                                          c * 8);
    *reinterpret_cast<uint4*>(dst + sw(r, c, D * 2)) = v;
  }
}

template <int D, bool BF16, int MASK, bool ALIBI>
__global__ void __launch_bounds__(kThreads, 1) bwd_main_kernel(const BwdArgs a) {
  using L = BSmem<D, BF16>;
  constexpr bool kCausal = (MASK == 1 || MASK == 3);
  constexpr bool kPacked = (MASK >= 2);
  constexpr int kHalf = D / 2;       // gradient dims per warp
  constexpr int kNT = kHalf / 8;     // n-tiles of 8 dims per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  float* s_lse = reinterpret_cast<float*>(smem + L::kLse);
  float* s_delta = reinterpret_cast<float*>(smem + L::kDelta);
  const uint32_t sbase = smem_u32(smem);

  const int nb = blockIdx.x, kvh = blockIdx.y, unit = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int wr = warp & 3, wc = warp >> 2;

  int q0 = 0, q_len = a.M, k0 = 0, k_len = a.N, bidx = unit;
  if constexpr (kPacked) {
    q0 = a.seqstart_q[unit];
    q_len = a.seqstart_q[unit + 1] - q0;
    k0 = a.seqstart_k[unit];
    k_len = a.seqstart_k[unit + 1] - k0;
    bidx = 0;
    if (q_len < 0 || k_len < 0 || q0 < 0 || k0 < 0 || q0 + q_len > a.M || k0 + k_len > a.N ||
        (nb == a.num_kblocks - 1 && k_len > a.num_kblocks * kBT)) {
      if (threadIdx.x == 0) record_error(a.status, kErrInvalidArg);
      return;
    }
  }
  const int n0 = nb * kBT;
  if (n0 >= k_len) return;
  const int off = k_len - q_len;

  // K and V rows of this block, kept for the whole CTA.
  const long long kv_row_stride = static_cast<long long>(a.Hkv) * D;
  const long long q_row_stride = static_cast<long long>(a.Hq) * D;
  const uint16_t* kbase = static_cast<const uint16_t*>(a.k) + static_cast<long long>(bidx) * a.N * kv_row_stride;
  const uint16_t* vbase = static_cast<const uint16_t*>(a.v) + static_cast<long long>(bidx) * a.N * kv_row_stride;
  load_tile<D>(smem + L::kK, kbase, k0 + n0, k0 + k_len, kv_row_stride, kvh);
  load_tile<D>(smem + L::kV, vbase, k0 + n0, k0 + k_len, kv_row_stride, kvh);

  float dv_acc[kNT][4], dk_acc[kNT][4];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dv_acc[nt][e] = dk_acc[nt][e] = 0.f;

  // First query block whose rows can see this key block.
  int m_first = 0;
  if constexpr (kCausal) m_first = max(0, n0 - off) / kBT * kBT;

  for (int hh = 0; hh < a.group; ++hh) {
    const int h = kvh * a.group + hh;
    float slope_log2 = 0.f;
    if constexpr (ALIBI) slope_log2 = exp2f(-8.0f * static_cast<float>(h + 1) / a.Hq) * kLog2e;
    const uint16_t* qbase = static_cast<const uint16_t*>(a.q) + static_cast<long long>(bidx) * a.M * q_row_stride;
    const uint16_t* obase = static_cast<const uint16_t*>(a.dout) + static_cast<long long>(bidx) * a.M * q_row_stride;
    for (int m0 = m_first; m0 < q_len; m0 += kBT) {
      __syncthreads();  // the previous block's tiles are no longer read
      load_tile<D>(smem + L::kQ, qbase, q0 + m0, q0 + q_len, q_row_stride, h);
      load_tile<D>(smem + L::kDO, obase, q0 + m0, q0 + q_len, q_row_stride, h);
      if (threadIdx.x < kBT) {
        const int r = m0 + threadIdx.x;
        const long long li = (static_cast<long long>(bidx) * a.Hq + h) * a.M + q0 + r;
        s_lse[threadIdx.x] = r < q_len ? a.lse[li] : neg_inf();
        s_delta[threadIdx.x] = r < q_len ? a.delta[li] : 0.f;
      }
      __syncthreads();

      // ---- S = Q K^T and dP = dO V^T: rows 16wr.., keys 32wc.. -------------
      float sc[4][4], dp[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = dp[nt][e] = 0.f;
      {
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t aq[4], ad[4];
          const int arow = wr * 16 + (mi & 1) * 8 + rr, achunk = 2 * ks + (mi >> 1);
          ldsm_x4(sbase + L::kQ + sw(arow, achunk, L::kRow), aq);
          ldsm_x4(sbase + L::kDO + sw(arow, achunk, L::kRow), ad);
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            const int key = wc * 32 + np * 16 + (mi >> 1) * 8 + rr, bchunk = 2 * ks + (mi & 1);
            uint32_t bk[4], bv[4];
            ldsm_x4(sbase + L::kK + sw(key, bchunk, L::kRow), bk);
            ldsm_x4(sbase + L::kV + sw(key, bchunk, L::kRow), bv);
            mma16816<BF16>(sc[2 * np], aq, bk[0], bk[1]);
            mma16816<BF16>(sc[2 * np + 1], aq, bk[2], bk[3]);
            mma16816<BF16>(dp[2 * np], ad, bv[0], bv[1]);
            mma16816<BF16>(dp[2 * np + 1], ad, bv[2], bv[3]);
          }
        }
      }

      // ---- P = exp(s - lse) (masked -> 0), dS = P (dP - D); to shared -------
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = wr * 16 + gid + half * 8;
        const int i_loc = m0 + row;
        const float lse_l2 = s_lse[row] * kLog2e;
        const float dlt = s_delta[row];
        const bool row_ok = i_loc < q_len && s_lse[row] != neg_inf();
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          float p2[2], ds2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = wc * 32 + nt * 8 + 2 * tig + e;
            const int j_loc = n0 + key;
            bool vis = row_ok && j_loc < k_len;
            if (kCausal) vis = vis && j_loc <= i_loc + off;
            float y = sc[nt][half * 2 + e] * a.scale_log2 - lse_l2;
            if constexpr (ALIBI)
              y -= slope_log2 * fabsf(static_cast<float>(i_loc + off - j_loc));
            const float p = vis ? ex2(y) : 0.f;
            p2[e] = p;
            ds2[e] = p * (dp[nt][half * 2 + e] - dlt);
          }
          const int key0 = wc * 32 + nt * 8 + 2 * tig;
          const uint32_t o = sw(row, key0 >> 3, kBT * 2) + (key0 & 7) * 2;
          const uint32_t ph = pack2<BF16>(p2[0], p2[1]);
          const uint32_t dh = pack2<BF16>(ds2[0], ds2[1]);
          *reinterpret_cast<uint32_t*>(smem + L::kP + o) = ph;
          *reinterpret_cast<uint32_t*>(smem + L::kDS + o) = dh;
          if constexpr (BF16) {
            *reinterpret_cast<uint32_t*>(smem + L::kPlo + o) =
                pack2<BF16>(p2[0] - __uint_as_float(ph << 16), p2[1] - __uint_as_float(ph & 0xffff0000u));
            *reinterpret_cast<uint32_t*>(smem + L::kDSlo + o) =
                pack2<BF16>(ds2[0] - __uint_as_float(dh << 16), ds2[1] - __uint_as_float(dh & 0xffff0000u));
          }
        }
      }
      __syncthreads();

      // ---- dV += P^T dO, dK += dS^T Q: keys 16wr.., dims kHalf*wc.. ----------
      // ---- dQ += dS K: rows 16wr.., dims kHalf*wc.. --------------------------
      float dq[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
      {
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int part = 0; part < (BF16 ? 2 : 1); ++part) {
          const uint32_t pT = sbase + (part ? L::kPlo : L::kP);
          const uint32_t dsT = sbase + (part ? L::kDSlo : L::kDS);
#pragma unroll
          for (int ks = 0; ks < kBT / 16; ++ks) {
            // A = P^T / dS^T (keys x rows) through transposed loads of [row][key].
            uint32_t ap[4], ads[4], adq[4];
            const int trow = ks * 16 + (mi >> 1) * 8 + rr, tchunk = wr * 2 + (mi & 1);
            ldsm_x4_t(pT + sw(trow, tchunk, kBT * 2), ap);
            ldsm_x4_t(dsT + sw(trow, tchunk, kBT * 2), ads);
            // A = dS (rows x keys) for dQ.
            const int arow = wr * 16 + (mi & 1) * 8 + rr, achunk = 2 * ks + (mi >> 1);
            ldsm_x4(dsT + sw(arow, achunk, kBT * 2), adq);
#pragma unroll
            for (int np = 0; np < kNT / 2; ++np) {
              // B = dO, Q, K ([k rows][n dims]) through transposed loads.
              const int brow = ks * 16 + (mi & 1) * 8 + rr;
              const int bchunk = (kHalf * wc) / 8 + 2 * np + (mi >> 1);
              uint32_t bo[4], bq[4], bk[4];
              ldsm_x4_t(sbase + L::kDO + sw(brow, bchunk, L::kRow), bo);
              ldsm_x4_t(sbase + L::kQ + sw(brow, bchunk, L::kRow), bq);
              ldsm_x4_t(sbase + L::kK + sw(brow, bchunk, L::kRow), bk);
              mma16816<BF16>(dv_acc[2 * np], ap, bo[0], bo[1]);
              mma16816<BF16>(dv_acc[2 * np + 1], ap, bo[2], bo[3]);
              mma16816<BF16>(dk_acc[2 * np], ads, bq[0], bq[1]);
              mma16816<BF16>(dk_acc[2 * np + 1], ads, bq[2], bq[3]);
              mma16816<BF16>(dq[2 * np], adq, bk[0], bk[1]);
              mma16816<BF16>(dq[2 * np + 1], adq, bk[2], bk[3]);
            }
          }
        }
      }
      // dq rows of this block (valid rows only), scaled, into the fp32 accumulator.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = m0 + wr * 16 + gid + half * 8;
        if (r >= q_len) continue;
        float* dst = a.dq_acc + ((static_cast<long long>(bidx) * a.M + q0 + r) * a.Hq + h) * D +
                     kHalf * wc + 2 * tig;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          atomicAdd(dst + nt * 8, dq[nt][half * 2] * a.scale);
          atomicAdd(dst + nt * 8 + 1, dq[nt][half * 2 + 1] * a.scale);
        }
      }
    }
  }

  // ---- write dK (scaled) and dV of the valid keys -----------------------------
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int key = wr * 16 + gid + half * 8;
    if (n0 + key >= k_len) continue;
    const long long row = (static_cast<long long>(bidx) * a.N + k0 + n0 + key) * a.Hkv + kvh;
    uint32_t* dkp = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.dk) + row * D + kHalf * wc + 2 * tig);
    uint32_t* dvp = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.dv) + row * D + kHalf * wc + 2 * tig);
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      dkp[nt * 4] = pack2<BF16>(dk_acc[nt][half * 2] * a.scale, dk_acc[nt][half * 2 + 1] * a.scale);
      dvp[nt * 4] = pack2<BF16>(dv_acc[nt][half * 2], dv_acc[nt][half * 2 + 1]);
    }
  }
}

template <int D, bool BF16, int MASK, bool ALIBI>
cudaError_t launch_main(const BwdLaunch& L, cudaStream_t stream) {
  auto kern = bwd_main_kernel<D, BF16, MASK, ALIBI>;
  const int smem = BSmem<D, BF16>::kBytes + 128;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const BwdArgs& a = L.args;
  dim3 grid(a.num_kblocks, a.Hkv, a.num_units);
  kern<<<grid, kThreads, smem, stream>>>(a);
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

cudaError_t launch_bwd(const BwdLaunch& L, cudaStream_t stream) {
  if (L.head_dim == 64)
    return L.bf16 ? launch_all<64, true>(L, stream) : launch_all<64, false>(L, stream);
  if (L.head_dim == 128)
    return L.bf16 ? launch_all<128, true>(L, stream) : launch_all<128, false>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mea
