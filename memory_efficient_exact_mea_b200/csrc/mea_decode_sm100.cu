// mea_decode_sm100.cu -- one decode step against a packed, ragged KV cache.
//
// A decode step attends a single new query per sequence to every cached key of
// that sequence ("Transformer : comprendre l'entrainement et l'inference",
// section "Pre-remplissage et decodage"; "Transformerを実装して少し理解した気に
// なる会(その4)", section "KV Cache").  The work is bound by reading the cache,
// so the design goal is to stream every cached byte exactly once at full HBM
// bandwidth:
//   * the cache of sequence b is cut into fixed chunks of kDecodeChunk rows;
//     one CTA handles one (chunk, kv head, sequence) and computes the partial
//     state (max, sum, unnormalised output) of all G = Hq/Hkv query heads that
//     share that kv head, so each cached byte is read once for all G heads;
//   * one producer warp streams the chunk's key/value tiles with TMA into a
//     3-stage shared-memory ring (128-byte swizzled, 16 KB per 64-row tile);
//   * four consumer warps each take 16 rows of a tile and run the two thin
//     contractions on the tensor cores with mma.sync (keys x heads and
//     dims x heads, heads padded to 8), with the running max / running sum
//     of "FlashAttention (2022)", "Il trucco della softmax ...";
//   * a second kernel merges the chunk partials exactly by their log-sum-exp.
#include <math.h>


#include "mea.h"
#include "mea_internal.h"
#include "sm100.cuh"

namespace mea {
namespace {

constexpr int kBT = 64;            // cache rows per pipeline stage
constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;  // 16 rows of each stage per warp
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kMaxGroup = 8;       // query heads per kv head (MMA n = 8)
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct DSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = kBT * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBar = kStages * kStageBytes;
  static constexpr int kAbort = kBar + 2 * kStages * 8;
  static constexpr int kBytes = kAbort + 16 + 1024;
  // After the ring has drained, the combine buffers reuse the stage memory.
  static constexpr int kCombM = 0;
  static constexpr int kCombL = kCombM + kConsumerWarps * kMaxGroup * 4;
  static constexpr int kCombAcc = kCombL + kConsumerWarps * kMaxGroup * 4;
  static_assert(kCombAcc + kConsumerWarps * kMaxGroup * D * 4 <= kBar, "combine area");
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
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

// Byte offset of (row, 16-byte column chunk `c16` of the 64-element block `blk`)
// inside a TMA tile written with the 128-byte swizzle.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int dchunk) {
  const int blk = dchunk >> 3, c16 = dchunk & 7;
  return blk * DSmem<D>::kChunkBytes + row * 128 + ((c16 ^ (row & 7)) << 4);
}

template <int D, bool BF16, bool ALIBI>
__global__ void __launch_bounds__(kThreads, 2)
    decode_partial_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using L = DSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = a.kv_seqstart[b];
  const int n = a.kv_seqstart[b + 1] - t0;
  if (n < 0 || t0 < 0 || t0 + n > a.cache_rows ||
      (n + kDecodeChunk - 1) / kDecodeChunk > a.max_splits) {
    if (split == 0 && kvh == 0 && threadIdx.x == 0) record_error(a.status, kErrInvalidArg);
    return;
  }
  const int s0 = split * kDecodeChunk;
  if (s0 >= n) return;
  const int s1 = min(n, s0 + kDecodeChunk);
  const int ntiles = (s1 - s0 + kBT - 1) / kBT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const int gid = lane >> 2, tig = lane & 3;
  float m_run[2] = {neg_inf(), neg_inf()};  // heads 2*tig, 2*tig+1 (log2 units)
  float l_part[2] = {0.f, 0.f};
  float acc[D / 16][4];

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int i = 0;
      for (; i < ntiles; ++i) {
        const int slot = i % kStages;
        if (!mbar_wait(&empty[slot], ((i / kStages) & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(&full[slot], L::kStageBytes);
        uint8_t* st = smem + slot * L::kStageBytes;
        const int row = t0 + s0 + i * kBT;
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_3d(st + c * L::kChunkBytes, &tmK, &full[slot], c * 64, kvh, row);
          tma_load_3d(st + L::kTileBytes + c * L::kChunkBytes, &tmV, &full[slot], c * 64, kvh,
                      row);
        }
      }
      for (int j = max(0, i - kStages); j < i; ++j)
        mbar_wait_drain(&full[j % kStages], (j / kStages) & 1, a.status);
    }
  } else {
    // Q^T as the B operand (k = head dim, n = query head of this group).
    const int G = a.group;
    uint32_t qb[D / 16][2];
    {
      const uint16_t* qrow = static_cast<const uint16_t*>(a.q) +
                             (static_cast<long long>(b) * a.Hq + kvh * G + gid) * D;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tig) : 0u;
        qb[ks][1] =
            gid < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * tig) : 0u;
      }
    }
    float slope[2] = {0.f, 0.f};
    if constexpr (ALIBI) {
#pragma unroll
      for (int e = 0; e < 2; ++e)
        slope[e] = exp2f(-8.0f * static_cast<float>(kvh * G + 2 * tig + e + 1) / a.Hq) * kLog2e;
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;

    const uint32_t sbase = smem_u32(smem);
    for (int i = 0; i < ntiles; ++i) {
      const int slot = i % kStages;
      if (!mbar_wait_warp(&full[slot], (i / kStages) & 1, abort_flag, a.status)) break;
      const uint32_t kt = sbase + slot * L::kStageBytes;
      const uint32_t vt = kt + L::kTileBytes;

      // S^T (16 rows x 8 heads) = K_rows . Q^T
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = warp * 16 + (mi & 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t af[4];
          ldsm_x4(kt + swz<D>(row, 2 * ks + (mi >> 1)), af);
          mma16816<BF16>(sc, af, qb[ks][0], qb[ks][1]);
        }
      }
      // scale (+ ALiBi), mask rows past the chunk end, running max per head
      const int tok0 = s0 + i * kBT + warp * 16 + gid;  // position in the sequence
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tok0 + ((e >> 1) << 3);
        float v = sc[e] * a.scale_log2;
        if constexpr (ALIBI) v = fmaf(-slope[e & 1], static_cast<float>(n - 1 - tok), v);
        x[e] = tok < s1 ? v : neg_inf();
      }
      float alpha[2], msub[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(x[e], x[e + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[e], mx);
        alpha[e] = (m_new == m_run[e]) ? 1.f : ex2(m_run[e] - m_new);
        m_run[e] = m_new;
        msub[e] = (m_new == neg_inf()) ? 0.f : m_new;
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = ex2(x[e] - msub[e & 1]);
#pragma unroll
      for (int e = 0; e < 2; ++e) l_part[e] = l_part[e] * alpha[e] + p[e] + p[e + 2];
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        acc[mt][0] *= alpha[0];
        acc[mt][1] *= alpha[1];
        acc[mt][2] *= alpha[0];
        acc[mt][3] *= alpha[1];
      }
      // P^T as the B operand: transpose the (rows x heads) accumulator fragments.
      // bf16 keeps only 8 significant bits, so P goes in as P_hi + P_lo.
      const uint32_t ph0 = pack2<BF16>(p[0], p[1]);
      const uint32_t ph1 = pack2<BF16>(p[2], p[3]);
      const uint32_t pb0 = movmatrix_trans(ph0);
      const uint32_t pb1 = movmatrix_trans(ph1);
      uint32_t pl0 = 0u, pl1 = 0u;
      if constexpr (BF16) {
        pl0 = movmatrix_trans(pack2<BF16>(p[0] - __uint_as_float(ph0 << 16),
                                          p[1] - __uint_as_float(ph0 & 0xffff0000u)));
        pl1 = movmatrix_trans(pack2<BF16>(p[2] - __uint_as_float(ph1 << 16),
                                          p[3] - __uint_as_float(ph1 & 0xffff0000u)));
      }
      // O^T (dims x heads) += V^T . P^T
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = warp * 16 + (mi >> 1) * 8 + rr;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t af[4];
          ldsm_x4_trans(vt + swz<D>(row, 2 * mt + (mi & 1)), af);
          mma16816<BF16>(acc[mt], af, pb0, pb1);
          if constexpr (BF16) mma16816<BF16>(acc[mt], af, pl0, pl1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 4);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 8);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 16);
    }
  }
  __syncthreads();  // the ring has drained: its memory now holds the combine buffers

  float* comb_m = reinterpret_cast<float*>(smem + L::kCombM);
  float* comb_l = reinterpret_cast<float*>(smem + L::kCombL);
  float* comb_acc = reinterpret_cast<float*>(smem + L::kCombAcc);
  if (warp < kConsumerWarps) {
    if (gid == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        comb_m[warp * kMaxGroup + 2 * tig + e] = m_run[e];
        comb_l[warp * kMaxGroup + 2 * tig + e] = l_part[e];
      }
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int head = 2 * tig + (e & 1);
        const int dim = mt * 16 + gid + ((e >> 1) << 3);
        comb_acc[(warp * kMaxGroup + head) * D + dim] = acc[mt][e];
      }
  }
  __syncthreads();
  const int G = a.group;
  if (*abort_flag) {
    // A wait gave up (the status word holds the timeout): mark this split's
    // partials as failed so the merge writes no result built from them.
    if (threadIdx.x < G) {
      const long long row = static_cast<long long>(b) * a.Hq + kvh * G + threadIdx.x;
      a.part_lse[row * a.max_splits + split] = __int_as_float(0x7fc00000);
    }
    return;
  }

  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    const int g = idx / D, d = idx - g * D;
    float mx = neg_inf();
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, comb_m[w * kMaxGroup + g]);
    const float msub = (mx == neg_inf()) ? 0.f : mx;
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float wgt = ex2(comb_m[w * kMaxGroup + g] - msub);
      lsum += wgt * comb_l[w * kMaxGroup + g];
      o += wgt * comb_acc[(w * kMaxGroup + g) * D + d];
    }
    const long long row = static_cast<long long>(b) * a.Hq + kvh * G + g;
    a.part_o[(row * a.max_splits + split) * D + d] = lsum > 0.f ? o / lsum : 0.f;
    if (d == 0)
      a.part_lse[row * a.max_splits + split] = lsum > 0.f ? mx + __log2f(lsum) : neg_inf();
  }
}

// Exact merge of the chunk partials: lse = log2 sum_s 2^lse_s,
// out = sum_s 2^(lse_s - lse) o_s.  One warp per (sequence, query head).
template <int D, bool BF16>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeArgs a) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.B * a.Hq) return;
  const int b = row / a.Hq;
  const int t0 = a.kv_seqstart[b];
  const int n = a.kv_seqstart[b + 1] - t0;
  uint16_t* out = static_cast<uint16_t*>(a.out) + static_cast<long long>(row) * D;
  // The partial kernel's checks of this sequence's offsets: a sequence it
  // skipped has no partials, so its rows get out = 0 and lse = NaN (and the
  // status word the error) rather than whatever the workspace held.
  if (n < 0 || t0 < 0 || t0 + n > a.cache_rows ||
      static_cast<long long>(n) > static_cast<long long>(a.max_splits) * kDecodeChunk) {
    if (lane == 0 && row % a.Hq == 0) record_error(a.status, kErrInvalidArg);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) out[lane + 32 * i] = 0;
    if (lane == 0 && a.lse != nullptr) a.lse[row] = __int_as_float(0x7fc00000);
    return;
  }
  const int ns = n <= 0 ? 0 : (n + kDecodeChunk - 1) / kDecodeChunk;
  const float* pl = a.part_lse + static_cast<long long>(row) * a.max_splits;
  const float* po = a.part_o + static_cast<long long>(row) * a.max_splits * D;
  float mx = neg_inf();
  bool failed = false;  // a split whose partial kernel gave up
  for (int s = lane; s < ns; s += 32) {
    const float x = pl[s];
    failed |= x != x;
    mx = fmaxf(mx, x);
  }
  if (__any_sync(0xffffffffu, failed)) {
#pragma unroll
    for (int i = 0; i < D / 32; ++i) out[lane + 32 * i] = 0;
    if (lane == 0 && a.lse != nullptr) a.lse[row] = __int_as_float(0x7fc00000);
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float msub = (mx == neg_inf()) ? 0.f : mx;
  float wsum = 0.f;
  float o[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) o[i] = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = ex2(pl[s] - msub);
    wsum += w;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) o[i] = fmaf(w, po[s * D + lane + 32 * i], o[i]);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    const float v = o[i] * inv;
    if constexpr (BF16) {
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      out[lane + 32 * i] = *reinterpret_cast<uint16_t*>(&h);
    } else {
      __half h = __float2half_rn(v);
      out[lane + 32 * i] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
  if (lane == 0 && a.lse != nullptr)
    a.lse[row] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : neg_inf();
}

template <int D, bool BF16, bool ALIBI>
cudaError_t launch_t(const DecodeLaunch& L, cudaStream_t stream) {
  const DecodeArgs& a = L.args;
  if (a.max_splits > 0 && a.B > 0) {
    constexpr auto kern = decode_partial_kernel<D, BF16, ALIBI>;
    const int smem = DSmem<D>::kBytes;
    cudaError_t e = set_smem_once<kern>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.max_splits, a.Hkv, a.B);
    kern<<<grid, kThreads, smem, stream>>>(L.tmK, L.tmV, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int rows = a.B * a.Hq;
  if (rows > 0) {
    decode_merge_kernel<D, BF16><<<(rows + 3) / 4, 128, 0, stream>>>(a);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace

// ---------------------------------------------------------------------------
// Allocation-free decode: the split partials live in a fixed device array that
// belongs to this library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device

// Every device that loads this library holds this array until the process exits.
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_decode_scratch on the current device.  Host code cannot use
// the symbol itself (on the host it names a stand-in, not device memory), so the
// address is looked up on every call, with the caller's device current (the
// lookup is cheap, and a cached address would go stale if the device's context
// were torn down and created again).
cudaError_t noalloc_scratch(void** ptr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *ptr = p;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
  const int key = (L.head_dim == 128 ? 4 : 0) + (L.bf16 ? 2 : 0) + (L.alibi ? 1 : 0);
  if (L.head_dim != 64 && L.head_dim != 128) return cudaErrorInvalidValue;
  switch (key) {
    case 0: return launch_t<64, false, false>(L, stream);
    case 1: return launch_t<64, false, true>(L, stream);
    case 2: return launch_t<64, true, false>(L, stream);
    case 3: return launch_t<64, true, true>(L, stream);
    case 4: return launch_t<128, false, false>(L, stream);
    case 5: return launch_t<128, false, true>(L, stream);
    case 6: return launch_t<128, true, false>(L, stream);
    case 7: return launch_t<128, true, true>(L, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mea

// The allocation-free entry point (declared in mea.h).  It validates the size
// against the built-in scratch and then runs exactly the mea_decode path with
// that scratch as its workspace.
extern "C" int mea_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* kv_seqstart, void* out, float* lse, int B,
                                  int Hq, int Hkv, int K, int cache_rows, int max_kv_len,
                                  mea_dtype_t dtype, int alibi, float scale,
                                  cudaStream_t stream) {
  const size_t need = mea_decode_workspace_size(B, Hq, Hkv, K, max_kv_len);
  if (need > mea::kNoAllocScratchBytes) return MEA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (mea::noalloc_scratch(&scratch) != cudaSuccess) return MEA_ERR_CUDA;
  return mea_decode(q, k_cache, v_cache, kv_seqstart, out, lse, B, Hq, Hkv, K, cache_rows,
                    max_kv_len, dtype, alibi, scale, scratch, mea::kNoAllocScratchBytes, stream);
}
