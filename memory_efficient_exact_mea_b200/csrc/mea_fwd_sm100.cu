// mea_fwd_sm100.cu -- prefill attention for B200 (sm_100a): TMA + tcgen05 + TMEM.
//
// Computes out = softmax(Q K^T * scale + bias) V and lse per row, tile by tile
// with a running max and running sum, so the score matrix lives only in tensor
// memory, one 128x128 tile at a time ("FlashAttention (2022)", sections "L'idea:
// non scrivere mai la matrice intera" and "Il trucco della softmax che non ha
// bisogno di vedere tutto").  Masks (causal, block-diagonal) are generated from
// indices and fully masked key tiles are never loaded ("Come costruire
// Transformer efficienti in memoria con xFormers ...", "Applicare Attenzione
// Causale con Maschere Inferiori", "Utilizzare Sequenze di Lunghezza Variabile").
//
// CTA organisation (608 threads, one CTA per SM):
//   warps 0-7   softmax / rescale / epilogue for query tile 0 (TMEM lanes 0-127):
//               each warp on 16 lanes of its lane quarter, four threads per row
//               (a quarter of the columns each) in one warp
//   warps 8-15  the same for query tile 1 (rows +128)
//   warp  16    TMEM allocator; issues every MMA of query tile 0 (and, with P
//               written over S, of query tile 1 too, interleaved)
//   warp  17    separate-P layout: issues every MMA of query tile 1 (the two
//               tiles do not wait for each other); both issuers run their loops
//               warp-wide, elect.sync picking the lane that executes each
//               tcgen05.mma and tcgen05.commit
//   warp  18    the single TMA-issuing thread
// Tensor memory (512 columns): S0 | S1 (128 fp32 columns each, the scores of the
// current key tile; P = exp(S - m) as 16-bit pairs is written back over S, each
// 32-key chunk over its own 32 columns: fp16 P in the first 16, bf16 as P_hi in
// the first 16 and P_lo = P - P_hi in the last 16; the P.V MMA reads P straight
// from TMEM) | O0 | O1 (K columns each, the fp32 output accumulators).  At K = 64
// with fp16, P has columns of its own instead (S0 | S1 | P0 | P1 | O0 | O1 =
// 128 + 128 + 64 + 64 + 64 + 64), so each tile's next Q.K^T overlaps its softmax.
// Shared memory: Q0, Q1 (loaded once per unit; two such buffers in the persistent
// instances, which walk several units per CTA) and a ring of key/value tiles, all
// in the 128-byte-swizzled layout the TMA writes and the MMA descriptors read.
#include <math.h>

#include <atomic>
#include <type_traits>

#include "mea_internal.h"
#include "sm100.cuh"

namespace mea {
namespace {

constexpr int kModeDense = 0, kModeSparse = 1, kModeCache = 2;
constexpr int kBM = 128;        // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;        // keys per tile
constexpr int kThreads = 608;
constexpr int kMmaWarp = 16;   // + tile: warps 16 and 17 each issue one query tile's MMAs
constexpr int kTmaWarp = 18;
constexpr int kSoftmaxWarpsPerTile = 8;  // four threads per row, 16 rows per warp
constexpr uint32_t kTmemCols = 512;
constexpr float kTau = 8.0f;    // keep a stale row max while the new one exceeds it by < 2^8
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// QB: Q buffers (two query tiles each); persistent instances double-buffer Q.
template <int D, int QB>
struct Smem {
  static constexpr int kChunks = D / 64;          // 64-element (128-byte) column chunks
  static constexpr int kChunkBytes = kBM * 128;   // one chunk of a 128-row tile
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kSlots = (D == 128) ? 4 : 8;
  static constexpr int kQ = 0;
  static constexpr int kKV = QB * 2 * kTileBytes;
  static constexpr int kBar = kKV + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 * QB + 2 * kSlots + 2 + 8 + 2 + 1 + 2;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  // Packed causal batches: sequences by decreasing length, and where each query
  // block level starts in the unit ranks (see fwd_kernel).
  static constexpr int kMaxSeqs = 256, kMaxLevels = 64;
  static constexpr int kSeqOrder = kAbort + 4;                  // int16[kMaxSeqs]
  static constexpr int kLevelStart = kSeqOrder + 2 * kMaxSeqs;  // int32[kMaxLevels + 1]
  static constexpr int kBytes = kLevelStart + 4 * (kMaxLevels + 1) + 1024;  // + base alignment
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// A copy of x that the compiler cannot merge with other uses of x, so that x
// need not stay live in a register until this point.
__device__ __forceinline__ int opaque(int x) {
  int y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Pipeline timeline for performance work: built only with -DMEA_TRACE, it
// records clock64() at each pipeline event of the first kTraceCtas CTAs.
// Slots per CTA (step counters modulo 256): softmax tile t, its step n, event e
// -> t*4096 + n*16 + e; MMA thread, ring step l, event e -> 8192 + l*16 + e (one
// issuing thread) or 8192 + t*2048 + l*8 + e (one per tile); unit k (modulo 64),
// softmax tile t -> 12288 + k*4 + 2t (start), + 1 (epilogue done); TMA ring copy
// i (modulo 512) issued -> 12544 + 2i; Q load of unit k (modulo 64) -> 13568 + k;
// softmax warp w, step n: P published -> 13632 + w*256 + n; epilogue of unit k,
// tile t: O complete, O read, rows stored -> 17728 + k*8 + 4t + (0, 1, 2).
#ifdef MEA_TRACE
constexpr int kTraceCtas = 4;
constexpr int kTraceSlots = 18240;
__device__ long long g_trace[kTraceCtas * kTraceSlots];
#define MEA_TRACE_AT(slot)                                                         \
  do {                                                                             \
    if (blockIdx.x < kTraceCtas && (slot) < kTraceSlots)                           \
      g_trace[blockIdx.x * kTraceSlots + (slot)] = clock64();                      \
  } while (0)
// Per-CTA globaltimer stamps (all CTAs up to kCtaTraceMax): slot 0 entry, 1 first
// score tile of query tile 0 ready, 2 its key loop done, 3 its output stored,
// 4 the SM the CTA ran on.
constexpr int kCtaTraceMax = 4096;
__device__ long long g_cta_trace[kCtaTraceMax * 8];
#define MEA_CTA_AT(i)                                                              \
  do {                                                                             \
    if (blockIdx.x < kCtaTraceMax) {                                               \
      long long t_;                                                                \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                       \
      g_cta_trace[blockIdx.x * 8 + (i)] = t_;                                      \
      unsigned sm_;                                                                \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(sm_));                             \
      g_cta_trace[blockIdx.x * 8 + 4] = sm_;                                       \
    }                                                                              \
  } while (0)
#else
#define MEA_TRACE_AT(slot) \
  do {                     \
  } while (0)
#define MEA_CTA_AT(i) \
  do {                \
  } while (0)
#endif

// MODE kModeSparse: a block mask (one byte per 128-query x 128-key block)
// leaves out whole score tiles ("FlashAttention (2022)", "Cosa mostravano i
// numeri": the block-sparse variant); a left-out tile is neither loaded nor
// multiplied.
// MODE kModeCache: one prefill chunk against a KV cache ("Transformer :
// comprendre l'entrainement et l'inference", "Pre-remplissage et decodage" and
// "Un cache KV simple"): the chunk's queries attend to the cached rows
// [0, past) (tmK/tmV over the cache) and to the chunk's own new rows (tmKn/tmVn
// over the new keys/values) at positions past + r, and the CTAs copy the new
// rows into the cache at [past, past + n).  Nothing in the launch reads a cache
// row at or after past, so the copy races with no load.  The last tile of each
// region is shifted back to end at the region's end (its first columns, seen by
// an earlier tile or before row 0, are masked), so no row beyond a sequence's
// valid rows is ever loaded.
// Persistent instances (every instance without a block mask or a cache): one CTA
// per SM walks several units, with every pipeline counter running on across
// units, so the next unit's Q, K/V and first Q.K^T overlap the current unit's
// last steps and output epilogue.  The units are dealt out in a fixed order
// (round k of CTA c takes rank k * gridDim.x + c, or + gridDim.x - 1 - c in odd
// rounds), so the heaviest units of a causal launch, which come first in rank
// order, are spread over every SM.
template <int D, bool BF16, int MASK, bool ALIBI, int MODE>
constexpr bool kPersistent = MODE == kModeDense;

// Q buffers (two query tiles each): persistent instances at K = 64 double-buffer
// Q, so the next unit's Q lands during this unit's key loop; at K = 128 (no
// shared memory to spare) the one buffer is reloaded once this unit's last
// Q.K^T has completed.
template <int D, bool BF16, int MASK, bool ALIBI, int MODE>
constexpr int kQBuffers = (kPersistent<D, BF16, MASK, ALIBI, MODE> && D == 64) ? 2 : 1;

template <int D, bool BF16, int MASK, bool ALIBI, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKn,
               const __grid_constant__ CUtensorMap tmVn, const FwdArgs a) {
  constexpr bool SPARSE = (MODE == kModeSparse);
  constexpr bool kCache = (MODE == kModeCache);
  constexpr bool kPersist = kPersistent<D, BF16, MASK, ALIBI, MODE>;
  constexpr bool kCausal = (MASK == 1 || MASK == 3);
  constexpr bool kPacked = (MASK >= 2);
  // Causal instances without a cache walk a unit's key tiles from the diagonal
  // back to the first: keys nearer the query come first, and with ALiBi, whose
  // bias falls with distance, the first tile then holds (nearly always) the row's
  // largest logits, so the running max rarely moves afterwards and the output is
  // rarely rescaled.  Each query tile computes a suffix of the unit's steps.
  constexpr bool kDesc = kCausal && MODE == kModeDense;
  constexpr bool kSplitP = BF16;  // P.V as (P_hi + P_lo).V for bf16
  // With K = 64 and fp16, P gets TMEM columns of its own (S 2x128, P 2x64, O 2x64
  // = 512), so S_t is free as soon as the softmax has read it and the next
  // Q.K^T of the same tile runs during its softmax.  Otherwise P is written over S.
  constexpr bool kSepP = (D == 64) && !BF16;
  constexpr int QB = kQBuffers<D, BF16, MASK, ALIBI, MODE>;
  using L = Smem<D, QB>;
  // Softmax tile body specialised separately for masked and unmasked tiles.
  constexpr bool kTileCopies = !ALIBI && MODE == kModeDense && !kPacked;
  constexpr uint32_t kColP = kSepP ? 2 * kBN : 0;          // + t * (kSepP ? kBN/2 : kBN)
  constexpr uint32_t kColO = kSepP ? 2 * kBN + kBN : 2 * kBN;  // + t * D
  constexpr int S = L::kSlots;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sKV = smem + L::kKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;        // [QB]
  uint64_t* q_empty = bars + QB;  // [QB] Q buffer free again (persistent instances)
  uint64_t* kv_full = bars + 2 * QB;
  uint64_t* kv_empty = bars + 2 * QB + S;
  uint64_t* s_full = bars + 2 * QB + 2 * S;
  // p_ready[4t + C]: P of tile t published; with P written over S, C counts its
  // 32-key chunks (the P.V MMAs of a chunk go out once it is published); the
  // separate-P layout publishes the whole tile on p_ready[4t].
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 8;
  uint64_t* mma_done = o_done + 2;
  uint64_t* s_free = mma_done + 1;    // S_t read out by the softmax (separate-P layout)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) MEA_CTA_AT(0);

  // ---- units: (query block, head, batch or sequence) ------------------------
  // A unit is two 128-row query tiles of one (head, batch or sequence); rank r
  // numbers the units.  Without a causal mask the query block varies fastest,
  // so the blocks of one (head, batch) -- and the heads sharing a key/value
  // head -- run together and read each K/V tile from L2 instead of DRAM.  Under
  // a causal mask a unit's work grows with its query block, so the ranks go by
  // query block, last (longest rows) first, with the heads fastest: the longest
  // units of the whole launch start first.
  // Packed batches under a causal mask: most units of the rank space above
  // would be empty (a short sequence has no late query blocks), and a fixed
  // order that skips empty ranks spreads the real ones unevenly.  There the
  // CTA first sorts the sequences by decreasing length (up to kMaxSeqs of them)
  // and ranks only units that exist: level l (query block num_mblocks - 1 - l)
  // holds the sequences longer than that block's first row, longest first,
  // heads fastest.  A sequence whose offsets are invalid is recorded in the
  // status word and gets no units.
  int16_t* seq_order = reinterpret_cast<int16_t*>(smem + L::kSeqOrder);
  int* level_start = reinterpret_cast<int*>(smem + L::kLevelStart);
  constexpr bool kCompactable = kPacked && kCausal;
  const bool compact =
      kCompactable && a.num_units <= L::kMaxSeqs && a.num_mblocks <= L::kMaxLevels;
  // Chunked prefill: a unit's work is its sequence's cached rows plus the new
  // ones, which differ widely between sequences, so the sequences are ranked by
  // that (decreasing, up to kMaxSeqs of them) and the units of the longest go
  // first; within a sequence as elsewhere (causal: last query block first).
  const bool by_keys = kCache && a.num_units <= L::kMaxSeqs;
  if constexpr (kCache) {
    if (by_keys) {
      auto keys_of = [&](int s) -> int { return a.cache_len[s] + (a.q_lens ? a.q_lens[s] : a.M); };
      for (int i = threadIdx.x; i < a.num_units; i += kThreads) {
        const int ki = keys_of(i);
        int pos = 0;
        for (int j = 0; j < a.num_units; ++j) {
          const int kj = keys_of(j);
          pos += (kj > ki) || (kj == ki && j < i);
        }
        seq_order[pos] = static_cast<int16_t>(i);
      }
      __syncthreads();
    }
  }
  if constexpr (kCompactable) {
    if (compact) {
      auto rows_of = [&](int s) -> int {  // query rows of sequence s; 0 if its offsets are invalid
        const int qs = a.seqstart_q[s], ql = a.seqstart_q[s + 1] - qs;
        const int ks = a.seqstart_k[s], kl = a.seqstart_k[s + 1] - ks;
        const bool bad = ql < 0 || kl < 0 || qs < 0 || ks < 0 || qs + ql > a.M ||
                         ks + kl > a.N || ql > a.num_mblocks * kFwdRowsPerCta;
        return bad ? -1 : ql;
      };
      for (int i = threadIdx.x; i < a.num_units; i += kThreads) {
        const int li = rows_of(i);
        if (li < 0) record_error(a.status, kErrInvalidArg);
        int pos = 0;
        for (int j = 0; j < a.num_units; ++j) {
          const int lj = rows_of(j);
          pos += (lj > li) || (lj == li && j < i);
        }
        seq_order[pos] = static_cast<int16_t>(i);
      }
      for (int l = threadIdx.x; l < a.num_mblocks; l += kThreads) {
        const int first_row = (a.num_mblocks - 1 - l) * kFwdRowsPerCta;
        int c = 0;
        for (int j = 0; j < a.num_units; ++j) c += rows_of(j) > first_row;
        level_start[l + 1] = c * a.Hq;  // units of level l, summed below
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        level_start[0] = 0;
        for (int l = 0; l < a.num_mblocks; ++l) level_start[l + 1] += level_start[l];
      }
      __syncthreads();
    }
  }
  int n_ranks = a.num_mblocks * a.Hq * a.num_units;
  if constexpr (kCompactable) {
    if (compact) n_ranks = level_start[a.num_mblocks];
  }
  int mb = 0, h = 0, unit = 0, kvh = 0, bidx = 0, m_base = 0;
  int q0 = 0, q_len = a.M, k0 = 0, k_len = a.N, off = 0;
  int past = 0;  // cache mode: rows cached before this chunk
  int n_past_tiles = 0, n_new_tiles = 0;
  int nt_tile[2] = {0, 0};  // key tiles each query tile computes
  int nt = 0;               // key tiles loaded (the larger of the two)
  const uint8_t* mrow0 = nullptr;  // block-sparse: the two query tiles' mask rows
  const uint8_t* mrow1 = nullptr;
  // Moves every per-unit value to unit `rank`.  Returns 0 if the unit's sequence
  // offsets are invalid (the status word records it; nothing to do), 1 if the
  // unit has no query rows, 2 if it has rows to compute.
  auto set_unit = [&](int rank) -> int {
    if (kCompactable && compact) {
      int l = 0;
      while (rank >= level_start[l + 1]) ++l;
      const int i = rank - level_start[l];
      h = i % a.Hq;
      unit = seq_order[i / a.Hq];
      mb = a.num_mblocks - 1 - l;
    } else if (kCache && by_keys) {
      const int per = a.Hq * a.num_mblocks;
      const int pos = rank / per;
      const int rem = rank - pos * per;
      unit = seq_order[pos];
      if (kCausal) {
        h = rem % a.Hq;
        mb = a.num_mblocks - 1 - rem / a.Hq;
      } else {
        mb = rem % a.num_mblocks;
        h = rem / a.num_mblocks;
      }
    } else if constexpr (kCausal) {
      const int per = a.Hq * a.num_units;
      const int level = rank / per;
      const int rem = rank - level * per;
      h = rem % a.Hq;
      unit = rem / a.Hq;
      mb = a.num_mblocks - 1 - level;
    } else {
      mb = rank % a.num_mblocks;
      const int rem = rank / a.num_mblocks;
      h = rem % a.Hq;
      unit = rem / a.Hq;
    }
    kvh = h / a.group;
    bidx = unit;
    if constexpr (kPacked) {
      q0 = a.seqstart_q[unit];
      q_len = a.seqstart_q[unit + 1] - q0;
      k0 = a.seqstart_k[unit];
      k_len = a.seqstart_k[unit + 1] - k0;
      bidx = 0;
      const bool bad = q_len < 0 || k_len < 0 || q0 < 0 || k0 < 0 || q0 + q_len > a.M ||
                       k0 + k_len > a.N || (mb == a.num_mblocks - 1 &&
                                            q_len > a.num_mblocks * kFwdRowsPerCta);
      if (bad) {
        if (threadIdx.x == 0) record_error(a.status, kErrInvalidArg);
        return 0;
      }
    }
    if constexpr (kCache) {
      past = a.cache_len[unit];
      q_len = a.q_lens ? a.q_lens[unit] : a.M;
      if (past < 0 || q_len < 0 || q_len > a.M || past > a.cap - q_len) {
        if (threadIdx.x == 0) record_error(a.status, kErrInvalidArg);
        return 0;
      }
      k_len = past + q_len;
    }
    m_base = mb * kFwdRowsPerCta;
    if (m_base >= q_len) return 1;
    off = k_len - q_len;  // bottom-right causal alignment
    // Key tiles each query tile needs.  Cache mode: the past tiles (all visible)
    // then the new tiles (up to the diagonal under a causal mask).
    n_past_tiles = kCache ? (past + kBN - 1) / kBN : 0;
    n_new_tiles = kCache ? (q_len + kBN - 1) / kBN : 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int mt = m_base + t * kBM;
      int nkeys = 0;
      if (mt < q_len) {
        nkeys = k_len;
        if (kCausal) nkeys = min(k_len, max(0, mt + kBM + off));
      }
      nt_tile[t] = (nkeys + kBN - 1) / kBN;
      if constexpr (kCache) {
        const int nn = mt < q_len ? (kCausal ? min(q_len, mt + kBM) : q_len) : 0;
        nt_tile[t] = mt < q_len ? n_past_tiles + (nn + kBN - 1) / kBN : 0;
      }
    }
    nt = max(nt_tile[0], nt_tile[1]);
    if constexpr (SPARSE) {
      const long long base = unit * a.bm_sb + static_cast<long long>(h) * a.bm_sh;
      mrow0 = a.block_mask + base + static_cast<long long>(2 * mb) * a.bm_nk;
      mrow1 = mrow0 + a.bm_nk;
    }
    return 2;
  };
  // Round k of this CTA: rank k * gridDim.x + c, or + gridDim.x - 1 - c in odd
  // rounds (persistent instances); the CTA's own rank otherwise.
  auto rank_of = [&](int k) -> int {
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return k * G + ((k & 1) ? G - 1 - c : c);
  };
  // Calls body() for each unit with query rows this CTA runs, in order, until
  // body() returns false.  Every role walks the same units.
  auto for_each_unit = [&](auto&& body) {
    if constexpr (kPersist) {
      for (int k = 0;; ++k) {
        const int r = rank_of(k);
        if (r >= n_ranks) return;
        if (set_unit(r) != 2) continue;
        if (!body(k)) return;
      }
    } else {
      body(0);  // the CTA's unit, set below
    }
  };

  if constexpr (!kPersist) {
    const int st = set_unit(static_cast<int>(blockIdx.x));
    if (st == 0) return;
    if constexpr (kCache) {
      // The append: the CTAs of one (sequence, kv head) -- its query heads times
      // its query blocks -- each copy an equal share of the new rows.
      const int slices = a.group * a.num_mblocks;
      const int slice = (h % a.group) * a.num_mblocks + mb;
      const long long r0 = static_cast<long long>(q_len) * slice / slices;
      const long long r1 = static_cast<long long>(q_len) * (slice + 1) / slices;
      constexpr int kPieces = D / 8;  // 16-byte pieces per row
      for (long long e = threadIdx.x; e < (r1 - r0) * kPieces * 2; e += kThreads) {
        const int kv = static_cast<int>(e & 1);
        const long long r = r0 + (e >> 1) / kPieces;
        const int c = static_cast<int>((e >> 1) % kPieces);
        const long long* ns = kv ? a.vn_s : a.kn_s;
        const long long* cs = kv ? a.vc_s : a.kc_s;
        const uint4* src = reinterpret_cast<const uint4*>(
            static_cast<const uint16_t*>(kv ? a.v_new : a.k_new) + unit * ns[0] + r * ns[1] +
            kvh * ns[2] + c * 8);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(kv ? a.v_cache : a.k_cache) +
                                              unit * cs[0] + (past + r) * cs[1] + kvh * cs[2] +
                                              c * 8);
        *dst = *src;
      }
    }
    if (st == 1) return;
  }

  // Key tile j: the row its copy starts at (in the cache or in the new rows),
  // the key position of its column 0 and its first column not already seen by
  // an earlier tile (or not before row 0).  Only the last tile of a region is
  // shifted back.
  struct KeyTile {
    int row, pos, lo;
    bool fresh;
  };
  auto key_tile = [&](int j) -> KeyTile {
    if constexpr (kCache) {
      if (j < n_past_tiles) {
        const bool last = j == n_past_tiles - 1;
        const int r = last ? past - kBN : j * kBN;
        return {r, r, last ? n_past_tiles * kBN - past : 0, false};
      }
      const int m = j - n_past_tiles;
      const bool last = m == n_new_tiles - 1;
      const int r = last ? q_len - kBN : m * kBN;
      return {r, past + r, last ? n_new_tiles * kBN - q_len : 0, true};
    }
    const int jk = kDesc ? nt - 1 - j : j;  // the key tile of step j
    return {k0 + jk * kBN, jk * kBN, 0, false};
  };

  // Does query tile t compute key tile j?  Every role walks the key tiles in
  // the same order and skips those neither query tile needs; the barriers of a
  // query tile count only the key tiles that tile computes.
  auto uses = [&](int t, int j) -> bool {
    if constexpr (kDesc) return j >= nt - nt_tile[t];
    if (j >= nt_tile[t]) return false;
    if constexpr (SPARSE) return __ldg(t ? mrow1 + j : mrow0 + j) != 0;
    return true;
  };

  // ---- set-up -----------------------------------------------------------
  if (threadIdx.x == 0) {
    for (int qb = 0; qb < QB; ++qb) {
      mbar_init(&q_full[qb], 1);
      mbar_init(&q_empty[qb], kSepP ? 2 : 1);  // one commit per MMA-issuing thread
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], kSepP ? 2 : 1);  // one release per MMA-issuing thread
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      for (int c = 0; c < 4; ++c) mbar_init(&p_ready[4 * t + c], kSoftmaxWarpsPerTile);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(mma_done, kSepP ? 2 : 1);
    for (int t = 0; t < 2; ++t) mbar_init(&s_free[t], kSoftmaxWarpsPerTile);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if constexpr (kCache) {
      tma_prefetch_desc(&tmKn);
      tma_prefetch_desc(&tmVn);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kTmaWarp) {
    // ===================== TMA producer =====================================
    // Per unit: its two Q tiles into Q buffer (unit count) % QB, then its K and V
    // tiles through the ring; the ring and unit counters run on across units.
    if (lane == 0) {
      int it = 0, iu = 0;  // K/V ring copies and Q loads, over all units
      for_each_unit([&](int) -> bool {
        if (nt == 0) return true;  // rows that see no key: nothing to load
        const int qb = iu % QB;
        // The buffer's previous unit (QB units back) has finished its Q.K^T MMAs.
        if (iu >= QB && !mbar_wait(&q_empty[qb], (iu / QB - 1) & 1, abort_flag, a.status))
          return false;
        mbar_arrive_expect_tx(&q_full[qb], 2 * L::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sQ + (2 * qb + t) * L::kTileBytes + c * L::kChunkBytes, &tmQ, &q_full[qb],
                        c * 64, h, q0 + m_base + t * kBM, bidx);
        MEA_TRACE_AT(13568 + (iu & 63));
        ++iu;
        for (int j = 0; j < nt; ++j) {
          if constexpr (SPARSE) {
            if (!uses(0, j) && !uses(1, j)) continue;
          }
          const KeyTile kt = key_tile(j);
          for (int kv = 0; kv < 2; ++kv, ++it) {
            const int slot = it % S;
            if (!mbar_wait(&kv_empty[slot], ((it / S) & 1) ^ 1, abort_flag, a.status)) break;
            mbar_arrive_expect_tx(&kv_full[slot], L::kTileBytes);
            const CUtensorMap* map = kv ? &tmV : &tmK;
            if (kCache && kt.fresh) map = kv ? &tmVn : &tmKn;
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_4d(sKV + slot * L::kTileBytes + c * L::kChunkBytes, map, &kv_full[slot],
                          c * 64, kvh, kt.row, bidx);
            MEA_TRACE_AT(12544 + (it & 511) * 2);
          }
          if (*abort_flag) return false;
        }
        return *abort_flag == 0;
      });
      // Let every copy this thread started land before the CTA can exit.
      for (int i = max(0, iu - QB); i < iu; ++i)
        mbar_wait_drain(&q_full[i % QB], (i / QB) & 1, a.status);
      for (int i = max(0, it - S); i < it; ++i)
        mbar_wait_drain(&kv_full[i % S], (i / S) & 1, a.status);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ===================== MMA issuers, one per query tile ====================
    // The whole warp runs the issuing loop (all values warp-uniform); elect.sync
    // picks the lane that issues each MMA and commit.
    const int tile = warp - kMmaWarp;
    {
      const uint32_t idesc_qk = idesc_f16(BF16, kBM, kBN, false);
      const uint32_t idesc_pv = idesc_f16(BF16, kBM, D, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      // S_t = Q_t K^T: both operands K-major; step k advances 16 elements (32 bytes)
      // inside a 128-byte swizzle row, then to the next 64-column chunk.
      auto issue_qk = [&](int t, int slot, uint32_t q_buf) {
        const uint32_t d = tmem_base + t * kBN;
        const uint32_t qa = q_buf + t * L::kTileBytes;
        const uint32_t kb = kv_addr + slot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
          umma_ss_warp(d, sdesc_sw128(qa + o, 16, 1024), sdesc_sw128(kb + o, 16, 1024), idesc_qk,
                  kk > 0);
        }
      };
      // O_t (+)= P_t V with P read from TMEM (two 16-bit elements per column) and V
      // N-major, its 64-column chunks L::kChunkBytes apart; step k covers 16 keys =
      // 2048 bytes of V.  Separate-P layout: keys 2c, 2c+1 in column c of P_t.
      auto issue_pv = [&](int t, int slot, bool accumulate) {
        const uint32_t d = tmem_base + kColO + t * D;
        const uint32_t p = tmem_base + kColP + t * (kBN / 2);
        const uint32_t vb = kv_addr + slot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ts_warp(d, p + kk * 8, sdesc_sw128(vb + kk * 2048, L::kChunkBytes, 1024), idesc_pv,
                  (accumulate || kk > 0) ? 1u : 0u);
      };
      // P over S: keys 32c..32c+31 in columns 32c..32c+15 (bf16: P_hi there and
      // P_lo = P - P_hi in the 16 columns after, through the same V descriptors).
      // The MMAs of each 32-key chunk go out as soon as the softmax has published
      // that chunk, so the contraction runs alongside the rest of the tile's softmax.
      auto pv_chunks = [&](int t, int slot, bool accumulate, uint32_t parity) -> bool {
        const uint32_t d = tmem_base + kColO + t * D;
        const uint32_t p = tmem_base + kColP + t * kBN;
        const uint32_t vb = kv_addr + slot * L::kTileBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (!mbar_wait_warp(&p_ready[4 * t + c], parity, abort_flag, a.status)) return false;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < (kSplitP ? 2 : 1); ++part)
#pragma unroll
            for (int kk = 2 * c; kk < 2 * c + 2; ++kk)
              umma_ts_warp(d, p + c * 32 + part * 16 + (kk & 1) * 8,
                      sdesc_sw128(vb + kk * 2048, L::kChunkBytes, 1024), idesc_pv,
                      (accumulate || kk > 0 || part > 0) ? 1u : 0u);
        }
        return true;
      };

      // Ring index 2j holds K_j, 2j+1 holds V_j; each slot is released when both
      // tiles' MMAs reading it have completed (two commits).  A key tile beyond
      // this query tile's range is still waited for, so the release keeps its order.
      // Per tile the order is Q.K_j^T, then P.V of the tile the softmax has
      // finished: V_{j-1} in the separate-P layout (Q.K_j^T only needs S_t read out),
      // V_j when P is written over S (Q.K_{j+1}^T must follow P.V_j).
      // li counts the key tiles in the ring (both query tiles), c the key tiles
      // this query tile has computed (its barrier phases).
      const int t = tile;
      auto pv_step = [&](int lv, bool used, int cu, bool acc) -> bool {
        const int vs = (2 * lv + 1) % S;
        if (!mbar_wait_warp(&kv_full[vs], ((2 * lv + 1) / S) & 1, abort_flag, a.status)) return false;
        MEA_TRACE_AT(8192 + t * 2048 + (lv & 255) * 8 + 2);
        if (used) {
          if (!mbar_wait_warp(&p_ready[4 * t], cu & 1, abort_flag, a.status)) return false;
          MEA_TRACE_AT(8192 + t * 2048 + (lv & 255) * 8 + 3);
          tc_fence_after();
          issue_pv(t, vs, acc);
          umma_commit_warp(&o_done[t]);
          MEA_TRACE_AT(8192 + t * 2048 + (lv & 255) * 8 + 4);
        }
        umma_commit_warp(&kv_empty[vs]);
        return true;
      };
      // Separate-P layout: one thread per query tile.  P.V stays one step behind
      // Q.K^T, over unit boundaries too, so the next unit's first Q.K^T goes out
      // before this unit's last P.V.
      if constexpr (kSepP) {
        bool ok = true, prev_used = false, prev_acc = false;
        // li: key tiles in the ring, c: key tiles this query tile computed (its
        // barrier phases), both over all units; iu: units with keys so far.
        int li = 0, c = 0, prev_c = 0, iu = 0;
        for_each_unit([&](int) -> bool {
          if (nt == 0) return true;
          const int qb = iu % QB;
          if (!(ok = mbar_wait_warp(&q_full[qb], (iu / QB) & 1, abort_flag, a.status))) return false;
          const uint32_t q_buf = q_addr + 2 * qb * L::kTileBytes;
          const int li0 = li, c0 = c;
          for (int j = 0; j < nt && ok; ++j) {
            const bool used = uses(t, j);
            if constexpr (SPARSE) {
              if (!used && !uses(1 - t, j)) continue;
            } else {
              // dense: every key tile is in the ring and a tile uses a prefix of the
              // steps (a suffix when walking down from the diagonal)
              li = li0 + j;
              c = c0 + (kDesc ? max(0, j - (nt - nt_tile[t])) : j);
            }
            const int ks = (2 * li) % S;
            if (!(ok = mbar_wait_warp(&kv_full[ks], ((2 * li) / S) & 1, abort_flag, a.status))) break;
            MEA_TRACE_AT(8192 + t * 2048 + (li & 255) * 8 + 0);
            if (used) {
              if (c > 0) {  // the softmax has read the previous S_t out of TMEM
                if (!(ok = mbar_wait_warp(&s_free[t], (c - 1) & 1, abort_flag, a.status))) break;
                tc_fence_after();
              }
              issue_qk(t, ks, q_buf);
              umma_commit_warp(&s_full[t]);
              MEA_TRACE_AT(8192 + t * 2048 + (li & 255) * 8 + 1);
            }
            umma_commit_warp(&kv_empty[ks]);
            if (li >= 1) ok = pv_step(li - 1, prev_used, prev_c, prev_acc);
            prev_used = used;
            prev_acc = c > c0;  // P.V accumulates after the unit's first key tile
            prev_c = c;
            c += used ? 1 : 0;
            ++li;
          }
          if constexpr (!SPARSE) {
            li = li0 + nt;
            c = c0 + nt_tile[t];
          }
          // This unit's Q buffer is free once its Q.K^T MMAs have completed.
          if constexpr (kPersist) umma_commit_warp(&q_empty[qb]);
          ++iu;
          return ok;
        });
        if (ok && li > 0) pv_step(li - 1, prev_used, prev_c, prev_acc);
      }
      // When P is written over S the chain softmax -> P.V -> Q.K^T of a tile is
      // serial, so one thread (warp 16) issues both tiles in the interleaved
      // order Q0.K_j, P1.V_{j-1}, Q1.K_j, P0.V_j, which keeps the two tiles half a
      // step apart: one tile's softmax overlaps the other tile's MMAs.  The P1.V
      // lag runs on over unit boundaries: the next unit's Q0.K_0 goes out before
      // this unit's last P1.V (S_0 is free once P0.V of the last step is issued,
      // since the MMAs of one thread execute in issue order).
      if (!kSepP && tile == 0) {
        // li: key tiles in the ring; it: ring slots; c0, c1: key tiles computed by
        // query tile 0, 1 (their barrier phases); all over all units.
        int it = 0, vslot_prev = 0, li = 0, c0 = 0, c1 = 0, prev_c1 = 0, iu = 0;
        bool ok = true, prev_u1 = false, prev_acc1 = false;
        for_each_unit([&](int) -> bool {
          if (nt == 0) return true;
          const int qb = iu % QB;
          if (!(ok = mbar_wait_warp(&q_full[qb], (iu / QB) & 1, abort_flag, a.status))) return false;
          const uint32_t q_buf = q_addr + 2 * qb * L::kTileBytes;
          const int li0 = li, c00 = c0, c10 = c1;
          for (int j = 0; j < nt && ok; ++j) {
            const bool u0 = uses(0, j), u1 = uses(1, j);
            if constexpr (SPARSE) {
              if (!u0 && !u1) continue;
            } else {  // dense: every key tile is in the ring and each tile uses a prefix
              li = li0 + j;  // (a suffix when walking down from the diagonal)
              it = 2 * li;
              c0 = c00 + (kDesc ? max(0, j - (nt - nt_tile[0])) : j);
              c1 = c10 + (kDesc ? max(0, j - (nt - nt_tile[1])) : j);
            }
            const int kslot = it % S;
            if (!(ok = mbar_wait_warp(&kv_full[kslot], (it / S) & 1, abort_flag, a.status))) break;
            MEA_TRACE_AT(8192 + (li & 255) * 16 + 0);
            ++it;
            if (u0) {
              issue_qk(0, kslot, q_buf);
              MEA_TRACE_AT(8192 + (li & 255) * 16 + 1);
              umma_commit_warp(&s_full[0]);
            }
            if (li >= 1) {  // P1.V of the previous ring step (maybe of the previous unit)
              if (prev_u1) {
                if (!(ok = pv_chunks(1, vslot_prev, prev_acc1, prev_c1 & 1))) break;
                MEA_TRACE_AT(8192 + (li & 255) * 16 + 2);
                umma_commit_warp(&o_done[1]);
              }
              umma_commit_warp(&kv_empty[vslot_prev]);
            }
            if (u1) {
              issue_qk(1, kslot, q_buf);
              MEA_TRACE_AT(8192 + (li & 255) * 16 + 3);
              umma_commit_warp(&s_full[1]);
            }
            // This unit's Q buffer is free once its last Q.K^T MMAs have completed.
            if (kPersist && j == nt - 1) umma_commit_warp(&q_empty[qb]);
            umma_commit_warp(&kv_empty[kslot]);
            const int vslot = it % S;
            if (!(ok = mbar_wait_warp(&kv_full[vslot], (it / S) & 1, abort_flag, a.status))) break;
            MEA_TRACE_AT(8192 + (li & 255) * 16 + 4);
            ++it;
            if (u0) {
              MEA_TRACE_AT(8192 + (li & 255) * 16 + 5);
              if (!(ok = pv_chunks(0, vslot, c0 > c00, c0 & 1))) break;
              MEA_TRACE_AT(8192 + (li & 255) * 16 + 6);
              umma_commit_warp(&o_done[0]);
              ++c0;
            }
            vslot_prev = vslot;
            prev_u1 = u1;
            prev_acc1 = c1 > c10;  // P.V accumulates after the unit's first key tile
            prev_c1 = c1;
            c1 += u1 ? 1 : 0;
            ++li;
          }
          if constexpr (!SPARSE) {
            li = li0 + nt;
            it = 2 * li;
            c0 = c00 + nt_tile[0];
            c1 = c10 + nt_tile[1];
          }
          ++iu;
          return ok;
        });
        if (ok && li > 0) {
          if (prev_u1 && pv_chunks(1, vslot_prev, prev_acc1, prev_c1 & 1)) umma_commit_warp(&o_done[1]);
          umma_commit_warp(&kv_empty[vslot_prev]);
        }
      }
      // Every MMA issued above has completed once this barrier flips.
      if (kSepP || tile == 0) {
        umma_commit_warp(mma_done);
        mbar_wait_drain(mma_done, 0, a.status);
      }
    }
  } else {
    // ===================== softmax warpgroups ===============================
    // Eight warps per query tile, each on 16 TMEM lanes of its lane quarter
    // (16-lane shapes): a thread holds rows lane0 + t1 and lane0 + t1 + 8 and, of
    // every 8-column group, the columns 2 t0 and 2 t0 + 1 (t0 = lane % 4,
    // t1 = lane / 4).  The four threads of a row are lanes 4 t1 .. 4 t1 + 3 of
    // one warp, so row maxima and row sums combine with two shuffles.  P goes
    // back as 16-bit pairs with the 16x128b shape, which puts keys 8k + 2 t0,
    // 8k + 2 t0 + 1 into column 4k + t0 of the packed block that the P.V MMA
    // reads: the separate P columns, or (P over S) each 32-key chunk's first 16
    // S columns, with bf16's P - P_hi in the chunk's last 16.
    const int t = warp >> 3;
    const int wt = warp & 7, quarter = wt & 3, hf = wt >> 2;
    const int t0 = lane & 3, t1 = lane >> 2;
    const int lane0 = quarter * 32 + hf * 16;
    const uint32_t lane_addr = static_cast<uint32_t>(lane0) << 16;
    const uint32_t s_addr = tmem_base + lane_addr + t * kBN;
    const uint32_t p_addr = tmem_base + lane_addr + kColP + t * (kSepP ? kBN / 2 : kBN);
    const uint32_t o_addr = tmem_base + lane_addr + kColO + t * D;
    constexpr int kOReg = D / 2;  // O registers of a thread: 2 rows x D/4 columns
    auto ld_o = [&](uint32_t(&o)[kOReg]) {
      if constexpr (D == 64) tmem_ld16x256_x8_wait(o_addr, o);
      else tmem_ld16x256_x16_wait(o_addr, o);
    };
    auto st_o = [&](const uint32_t(&o)[kOReg]) {
      if constexpr (D == 64) tmem_st16x256_x8(o_addr, o);
      else tmem_st16x256_x16(o_addr, o);
    };
    const bool tracer = wt == 0 && lane == 0;
    // One arrival per warp on the tile's barriers (counts kSoftmaxWarpsPerTile):
    // each thread has fenced its tensor-memory accesses (tcgen05.fence::
    // before_thread_sync) before the warp synchronises and one lane arrives.
    auto warp_arrive = [](uint64_t* bar) { mbar_arrive_warp(bar); };
    // A zero scale is taken as 1e-30 (the same softmax to fp32 precision for any
    // finite score), so that -inf * scale stays -inf for hidden keys.
    const float scale_log2 = fmaxf(a.scale_log2, 1e-30f);
    bool ok = true;
    int nc = 0;  // key tiles this query tile has computed, over all units (barrier phases)
    for_each_unit([&](int ku) -> bool {
      const int nbase = nc;  // nc at the unit's start
      if (tracer) MEA_TRACE_AT(12288 + (ku & 63) * 4 + 2 * t);
      const int ntt = nt_tile[t];
      int rr[2], pos[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        rr[e] = m_base + t * kBM + lane0 + t1 + 8 * e;  // row inside the sequence
        pos[e] = rr[e] + off;                           // its position in key coordinates
      }
      float slope_log2 = 0.f;
      if constexpr (ALIBI) slope_log2 = exp2f(-8.0f * static_cast<float>(h + 1) / a.Hq) * kLog2e;
      float m_ref[2] = {neg_inf(), neg_inf()};  // reference max per row (log2 units)
      float l_sum[2] = {0.f, 0.f};              // this thread's part of each row sum
      for (int j = 0; j < ntt; ++j) {
        if constexpr (SPARSE) {
          if (!uses(t, j)) continue;
        } else {
          nc = nbase + j;
        }
        if (!(ok = mbar_wait_warp(&s_full[t], nc & 1, abort_flag, a.status))) break;
        if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 0);
        if (tracer && t == 0 && j == 0 && ku == 0) MEA_CTA_AT(1);
        // Keys this row may see in the tile: columns [kfirst, limit).  Tiles that
        // need no masking for any row of the warp take the unmasked path.
        int n0 = (kDesc ? ntt - 1 - j : j) * kBN, kfirst = 0;
        if constexpr (kCache) {
          const KeyTile kt = key_tile(j);
          n0 = kt.pos;
          kfirst = kt.lo;
        }
        int limit[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          limit[e] = k_len - n0;
          if (kCausal) limit[e] = min(limit[e], pos[e] + 1 - n0);
        }
        const bool masked = __any_sync(0xffffffffu, limit[0] < kBN || limit[1] < kBN) ||
                            (kCache && kfirst > 0);
        auto hidden = [&](int col, int e) -> bool {
          if constexpr (kCache) return col >= limit[e] || col < kfirst;
          return col >= limit[e];
        };
        // The tile's softmax.  `msk` is std::true_type / std::false_type for a copy
        // specialised to masked / unmasked tiles, or a run-time bool for one copy that
        // branches inside (only pass 1 masks: it sets hidden scores to -inf).
        auto tile = [&](auto msk) -> bool {
          tc_fence_after();
          uint32_t sr[64];  // register 4k + 2e + c: row e, column 8k + 2 t0 + c
          tmem_ld16x256_x16_wait(s_addr, sr);
          if constexpr (kSepP) {
            tc_fence_before();
            warp_arrive(&s_free[t]);  // S_t may now be overwritten by the next Q.K^T
          }

          // ---- pass 1: row maxima (log2 units) --------------------------------------
          // ALiBi: the bias of column 8k + 2 t0 + c in row e is -slope |db[e] + 8k + c|,
          // recomputed in both passes (cheaper than keeping the biased logits live).
          // Under a causal mask a visible key is never after the query, so the bias
          // is linear in the column there: slope (db[e] + 8k + c); hidden columns are
          // set to -inf anyway.
          float db[2], sdb[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            db[e] = static_cast<float>(n0 + 2 * t0 - pos[e]);
            sdb[e] = slope_log2 * db[e];
          }
          auto bias = [&](int k, int c, int e) -> float {
            if constexpr (kCausal) return fmaf(slope_log2, static_cast<float>(8 * k + c), sdb[e]);
            return -slope_log2 * fabsf(db[e] + static_cast<float>(8 * k + c));
          };
          float mx[2] = {neg_inf(), neg_inf()};
          if constexpr (ALIBI) {
            auto biased = [&](auto bmsk) {
#pragma unroll
              for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                  for (int c = 0; c < 2; ++c) {
                    float y = fmaf(__uint_as_float(sr[4 * k + 2 * e + c]), scale_log2, bias(k, c, e));
                    if constexpr (decltype(bmsk)::value) {
                      if (hidden(8 * k + 2 * t0 + c, e)) y = neg_inf();
                    }
                    sr[4 * k + 2 * e + c] = __float_as_uint(y);  // the biased logit, for pass 2
                    mx[e] = fmaxf(mx[e], y);
                  }
            };
            if (masked) biased(std::true_type{});
            else biased(std::false_type{});
          } else {
            auto max_plain = [&] {
#pragma unroll
              for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                  mx[e] = max3(mx[e], __uint_as_float(sr[4 * k + 2 * e]),
                               __uint_as_float(sr[4 * k + 2 * e + 1]));
            };
            // Hidden scores become -inf, so pass 2 needs no mask: 2^(-inf * scale - m)
            // = 0 (scale_log2 > 0 here).
            auto max_masked = [&] {
#pragma unroll
              for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                  for (int c = 0; c < 2; ++c) {
                    if (hidden(8 * k + 2 * t0 + c, e)) sr[4 * k + 2 * e + c] = __float_as_uint(neg_inf());
                    mx[e] = fmaxf(mx[e], __uint_as_float(sr[4 * k + 2 * e + c]));
                  }
            };
            if (flag_on(msk)) max_masked();
            else max_plain();
          }
          float alpha[2], nsub[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float pm = mx[e];
            if constexpr (!ALIBI) pm *= scale_log2;
            pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 1));
            pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 2));
            float m_use = m_ref[e];
            if (pm > m_ref[e] + kTau) m_use = pm;  // also taken when m_ref is -inf
            alpha[e] = (m_use == m_ref[e]) ? 1.f : ex2(m_ref[e] - m_use);
            m_ref[e] = m_use;
            nsub[e] = (m_use == neg_inf()) ? 0.f : -m_use;
          }
          if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 1);
          // The warp's output rows need a rescale (not at a unit's first key tile,
          // whose P.V overwrites O).  Decided here with P over S, whose chunks are
          // published during pass 2 unless the warp rescales.
          auto need_rescale = [&] {
            return nc > nbase && __any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f);
          };
          [[maybe_unused]] bool resc = false;
          if constexpr (!kSepP) resc = need_rescale();

          // ---- pass 2: P = 2^(logit - m), partial row sums, 16-bit pairs ------------
          // Hidden logits are -inf by now (pass 1), so one mask-free copy serves every tile.
          f2 ps[2] = {{0.f, 0.f}, {0.f, 0.f}};
          const f2 scale2 = {scale_log2, scale_log2};
          auto pass2 = [&]() -> bool {
            auto p_pair = [&](int k, int e) -> f2 {
              const f2 v = {__uint_as_float(sr[4 * k + 2 * e]), __uint_as_float(sr[4 * k + 2 * e + 1])};
              const f2 ns = {nsub[e], nsub[e]};
              const f2 y = ALIBI ? add2(v, ns) : fma2(v, scale2, ns);  // ALiBi: v is the biased logit
              const f2 p = {ex2(y.x), ex2(y.y)};
              ps[e] = add2(ps[e], p);
              return p;
            };
            if constexpr (kSepP) {
              uint32_t pk[32];  // 16x128b order: register 2k + e = row e, keys 8k + 2 t0, +1
#pragma unroll
              for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const f2 p = p_pair(k, e);
                  pk[2 * k + e] = pack2<BF16>(p.x, p.y);
                }
              if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 2);
              // P_t is still being read by P.V of the previous key tile.
              if (nc > 0 && !mbar_wait_warp(&o_done[t], (nc - 1) & 1, abort_flag, a.status))
                return false;
              tc_fence_after();
              tmem_st16x128_x16(p_addr, pk);
            } else {
              // P over S, one 32-key chunk C (k = 4C .. 4C + 3) at a time: the hi pairs
              // are repetitions 0..3 of a 16x128b store at the chunk's column, bf16's
              // lo pairs repetitions 4..7.  Without a rescale, chunk C - 1 is published
              // once chunk C is computed (its store has landed by then); a warp that
              // rescales publishes every chunk after the rescale below.
#pragma unroll
              for (int C = 0; C < 4; ++C) {
                uint32_t pc[kSplitP ? 16 : 8];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                  for (int e = 0; e < 2; ++e) {
                    const f2 p = p_pair(4 * C + kk, e);
                    const uint32_t hi = pack2<BF16>(p.x, p.y);
                    pc[2 * kk + e] = hi;
                    if constexpr (kSplitP) {
                      const f2 hf2 = {__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u)};
                      const f2 res = fma2(hf2, f2{-1.f, -1.f}, p);  // P - P_hi, exact in fp32
                      pc[8 + 2 * kk + e] = pack2<BF16>(res.x, res.y);
                    }
                  }
                if (C > 0 && !resc) {
                  tmem_st_wait();
                  tc_fence_before();
                  warp_arrive(&p_ready[4 * t + C - 1]);
                }
                if constexpr (kSplitP) tmem_st16x128_x8(p_addr + 32 * C, pc);
                else tmem_st16x128_x4(p_addr + 32 * C, pc);
              }
              if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 2);
            }
            return true;
          };
          if (!pass2()) return false;
#pragma unroll
          for (int e = 0; e < 2; ++e) l_sum[e] = l_sum[e] * alpha[e] + (ps[e].x + ps[e].y);
          if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 3);
          // Rescale the output rows whose reference max moved (after the previous
          // P.V has written O).
          if constexpr (kSepP) resc = need_rescale();
          if (resc) {
            if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 6);
            if constexpr (!kSepP) {
              if (!mbar_wait_warp(&o_done[t], (nc - 1) & 1, abort_flag, a.status)) return false;
              tc_fence_after();
            }
            uint32_t o[kOReg];  // register 4k + 2e + c: row e, column 8k + 2 t0 + c
            ld_o(o);
#pragma unroll
            for (int k = 0; k < D / 8; ++k)
#pragma unroll
              for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int c = 0; c < 2; ++c)
                  o[4 * k + 2 * e + c] = __float_as_uint(__uint_as_float(o[4 * k + 2 * e + c]) * alpha[e]);
            st_o(o);
          }
          if constexpr (!kSepP) {  // publish what is left of P (the chunks above)
            tmem_st_wait();
            tc_fence_before();
            if (resc) {
#pragma unroll
              for (int c = 0; c < 3; ++c) warp_arrive(&p_ready[4 * t + c]);
            }
            warp_arrive(&p_ready[4 * t + 3]);
          }
          return true;
        };
        // Two specialised copies where that compiles best (no register spills in the
        // plain dense instances, measured); one copy elsewhere, and for ALiBi, whose
        // biased-logit pass branches on `masked` itself.
        if constexpr (kTileCopies) ok = masked ? tile(std::true_type{}) : tile(std::false_type{});
        else ok = tile(!ALIBI && masked);
        if (!ok) break;
        if constexpr (kSepP) {
          tmem_st_wait();
          tc_fence_before();
          warp_arrive(&p_ready[4 * t]);
        }
        if (tracer) MEA_TRACE_AT(t * 4096 + (nc & 255) * 16 + 4);
        if (lane == 0) MEA_TRACE_AT(13632 + (warp & 15) * 256 + (nc & 255));
        ++nc;
      }
      if constexpr (!SPARSE) nc = nbase + ntt;
      if (tracer && t == 0 && ku == 0) MEA_CTA_AT(2);

      // ---- epilogue: out = O / l, lse = (m + log2 l) * ln 2 ---------------------
      // (Persistent instances recompute the rows here rather than keep them in
      // registers through the key loop: that instance then compiles without spills.)
      if constexpr (kPersist) {
#pragma unroll
        for (int e = 0; e < 2; ++e) rr[e] = opaque(m_base + t * kBM + lane0 + t1 + 8 * e);
      }
      if (ok && nc > nbase) ok = mbar_wait_warp(&o_done[t], (nc - 1) & 1, abort_flag, a.status);
      if (tracer) MEA_TRACE_AT(17728 + (ku & 63) * 8 + 4 * t);
      if (ok) {
        tc_fence_after();
        float l_tot[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          l_tot[e] = l_sum[e] + __shfl_xor_sync(0xffffffffu, l_sum[e], 1);
          l_tot[e] += __shfl_xor_sync(0xffffffffu, l_tot[e], 2);
        }
        uint32_t o[kOReg];
        if (nc > nbase) {
          ld_o(o);
        } else {
#pragma unroll
          for (int i = 0; i < kOReg; ++i) o[i] = 0u;
        }
        if (tracer) MEA_TRACE_AT(17728 + (ku & 63) * 8 + 4 * t + 1);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (rr[e] >= q_len) continue;
          const float inv_l = l_tot[e] > 0.f ? 1.f / l_tot[e] : 0.f;
          uint8_t* orow = reinterpret_cast<uint8_t*>(a.out) +
                          2 * (bidx * a.o_sb + static_cast<long long>(q0 + rr[e]) * a.o_sm +
                               h * a.o_sh + 2 * t0);
#pragma unroll
          for (int k = 0; k < D / 8; ++k)
            *reinterpret_cast<uint32_t*>(orow + 16 * k) =
                pack2<BF16>(__uint_as_float(o[4 * k + 2 * e]) * inv_l,
                            __uint_as_float(o[4 * k + 2 * e + 1]) * inv_l);
          if (t0 == 0 && a.lse != nullptr) {
            const float lse = l_tot[e] > 0.f ? (m_ref[e] + __log2f(l_tot[e])) * kLn2 : neg_inf();
            a.lse[(static_cast<long long>(bidx) * a.Hq + h) * a.M + q0 + rr[e]] = lse;
          }
        }
      }
      if (tracer && t == 0 && ku == 0) MEA_CTA_AT(3);
      if (tracer) MEA_TRACE_AT(17728 + (ku & 63) * 8 + 4 * t + 2);
      if (tracer) MEA_TRACE_AT(12288 + (ku & 63) * 4 + 2 * t + 1);
      return ok;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Streaming multiprocessors of the current device (looked up once per device).
cudaError_t sm_count(int* out) {
  static std::atomic<int> cached[64];  // zero-initialised (static storage)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) {
    const int n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) {
      *out = n;
      return cudaSuccess;
    }
  }
  e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess && dev >= 0 && dev < 64) cached[dev].store(*out, std::memory_order_relaxed);
  return e;
}

template <int D, bool BF16, int MASK, bool ALIBI, int MODE = kModeDense>
cudaError_t launch_t(const FwdLaunch& L, cudaStream_t stream) {
  constexpr auto kern = fwd_kernel<D, BF16, MASK, ALIBI, MODE>;
  constexpr bool kPersist = kPersistent<D, BF16, MASK, ALIBI, MODE>;
  const int smem = Smem<D, kQBuffers<D, BF16, MASK, ALIBI, MODE>>::kBytes;
  cudaError_t e = set_smem_once<kern>(smem);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(L.args.num_mblocks) * L.args.Hq *
                         L.args.num_units;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  long long ctas = grid;
  if constexpr (kPersist) {
    int sms = 0;
    e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    ctas = min(grid, static_cast<long long>(sms));  // one CTA per SM
  }
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(L.tmQ, L.tmK, L.tmV, L.tmKn,
                                                                  L.tmVn, L.args);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t dispatch_mask(const FwdLaunch& L, cudaStream_t s) {
  if (L.args.block_mask != nullptr) {  // block-sparse: no mask or causal only
    switch (L.mask * 2 + (L.alibi ? 1 : 0)) {
      case 0: return launch_t<D, BF16, 0, false, kModeSparse>(L, s);
      case 1: return launch_t<D, BF16, 0, true, kModeSparse>(L, s);
      case 2: return launch_t<D, BF16, 1, false, kModeSparse>(L, s);
      case 3: return launch_t<D, BF16, 1, true, kModeSparse>(L, s);
    }
    return cudaErrorInvalidValue;
  }
  if (L.args.cache_len != nullptr) {  // prefill chunk against a cache: no mask or causal
    switch (L.mask * 2 + (L.alibi ? 1 : 0)) {
      case 0: return launch_t<D, BF16, 0, false, kModeCache>(L, s);
      case 1: return launch_t<D, BF16, 0, true, kModeCache>(L, s);
      case 2: return launch_t<D, BF16, 1, false, kModeCache>(L, s);
      case 3: return launch_t<D, BF16, 1, true, kModeCache>(L, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (L.mask * 2 + (L.alibi ? 1 : 0)) {
    case 0: return launch_t<D, BF16, 0, false>(L, s);
    case 1: return launch_t<D, BF16, 0, true>(L, s);
    case 2: return launch_t<D, BF16, 1, false>(L, s);
    case 3: return launch_t<D, BF16, 1, true>(L, s);
    case 4: return launch_t<D, BF16, 2, false>(L, s);
    case 5: return launch_t<D, BF16, 2, true>(L, s);
    case 6: return launch_t<D, BF16, 3, false>(L, s);
    case 7: return launch_t<D, BF16, 3, true>(L, s);
  }
  return cudaErrorInvalidValue;
}

__global__ void fill_empty_kernel(uint16_t* out, float* lse, int B, int M, int Hq, int K,
                                  long long o_sb, long long o_sm, long long o_sh) {
  const long long rows = static_cast<long long>(B) * M * Hq;
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long b = r / (static_cast<long long>(M) * Hq);
    const long long i = (r / Hq) % M;
    const long long h = r % Hq;
    uint16_t* row = out + b * o_sb + i * o_sm + h * o_sh;
    for (int d = 0; d < K; ++d) row[d] = 0;
    if (lse) lse[(b * Hq + h) * M + i] = neg_inf();
  }
}

}  // namespace

cudaError_t launch_fwd(const FwdLaunch& L, cudaStream_t stream) {
  if (L.head_dim == 64)
    return L.bf16 ? dispatch_mask<64, true>(L, stream) : dispatch_mask<64, false>(L, stream);
  if (L.head_dim == 128)
    return L.bf16 ? dispatch_mask<128, true>(L, stream) : dispatch_mask<128, false>(L, stream);
  return cudaErrorInvalidValue;
}

#ifdef MEA_TRACE
// Copies the recorded timeline (kTraceCtas x kTraceSlots clock64 values) to host.
extern "C" int mea_trace_read(long long* host, int n) {
  if (n > kTraceCtas * kTraceSlots) n = kTraceCtas * kTraceSlots;
  return cudaMemcpyFromSymbol(host, g_trace, n * sizeof(long long)) == cudaSuccess ? n : -1;
}

extern "C" int mea_trace_cta_read(long long* host, int n) {
  if (n > kCtaTraceMax * 8) n = kCtaTraceMax * 8;
  return cudaMemcpyFromSymbol(host, g_cta_trace, n * sizeof(long long)) == cudaSuccess ? n : -1;
}
#endif

cudaError_t launch_fill_empty(void* out, float* lse, int B, int M, int Hq, int K, long long o_sb,
                              long long o_sm, long long o_sh, cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * M * Hq;
  if (rows <= 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = min((rows + threads - 1) / threads, 4096LL);
  fill_empty_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<uint16_t*>(out), lse, B, M, Hq, K, o_sb, o_sm, o_sh);
  return cudaGetLastError();
}

}  // namespace mea
