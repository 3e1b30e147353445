// hylra_kernels.cuh - HyLRA decode-attention kernels for sm_100a.
//
// "HyLRA: Hybrid Layer Reuse Attention for Efficient Long-Context Inference"
// (gist.science technical summary of arXiv 2602.00777):
//   §2.3 Hybrid Inference Strategy - reset layers: full attention + top-k
//        extraction; reuse layers: attention restricted to the reused subset.
//   §2.4 Block-level Sparsity - 128-token blocks, regular coalesced access.
//
// Kernels:
//   * decode_bf16_kernel: one persistent CTA per SM, static "stream-K" split.
//     A unit of work is one 128-token block of one (sequence b, KV head h):
//     every block of the cache on a reset layer, the k' reused blocks on a
//     reuse layer.  Units are laid out (b, h, j)-major and CTA c takes a
//     contiguous range (part_lo: CTAs that start late, behind the preceding
//     kernel, take a few units fewer).  Each maximal run of one (b, h) in a
//     CTA is a "segment" and leaves one partial state in the workspace.  Warp
//     0 issues TMA tile loads (128-byte swizzle, L2 evict-first) of K and V
//     (64 KB per stage, 3 stages) plus the GQA group's q rows; eight consumer
//     warps take 16 tokens each.  Q.K^T runs as S^T = K Q^T on bf16
//     mma.sync (M = tokens, N = the r <= 8 q-heads), the softmax is online in
//     the log2 domain with an fp32 running max and sum per warp, P^T moves
//     to the B-operand layout with movmatrix, and O^T = V^T P^T accumulates
//     in fp32 registers.  Reset layers also record, per block and q-head, the
//     block's local max and probability sum relative to it: the exact
//     ingredients of the block's attention mass once the global max and sum
//     are known.
//   * merge_kernel (reset layers) and merge_reuse_kernel (reuse layers): the
//     streaming kernel's programmatic dependent, per (b, h): LSE merge of the
//     segments' partials into the output and, on reset layers, the block
//     masses and the top-k (topk_select); on reuse layers the index-list
//     check.
//   * decode_reuse_cluster_kernel: a reuse layer as one thread-block
//     cluster per (b, h); the CTAs' states meet in CTA 0's shared memory
//     (st.async), which writes the output.
//   * gather_blocks_kernel: index-guided offloading, the reused blocks from
//     host memory into a device staging cache.
//   * decode_f32_kernel: fp32 inputs (small cases), CUDA cores, the same
//     split and records; the last CTA of a (b, h) (an atomic ticket, no
//     spinning) merges and selects in-kernel (merge_bh).
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "hylra.h"
#include "hylra_device.cuh"

namespace hylra {

constexpr int BLK = HYLRA_BLOCK_TOKENS;  // tokens per block
constexpr int HD = HYLRA_HEAD_DIM;       // head dimension
constexpr int GMAX = HYLRA_MAX_GROUP;    // q-heads per KV head, padded MMA N
constexpr int NW_BF16 = 8;               // consumer warps of the bf16 kernel (16 tokens each)
constexpr int NT_BF16 = NW_BF16 * 32;    // consumer threads of the bf16 kernel
constexpr int NTHR_BF16 = NT_BF16 + 32;  // + one producer warp
constexpr int NW_F32 = 4;                // warps of the fp32 kernel (32 tokens each)
constexpr int NT_F32 = NW_F32 * 32;
constexpr int NWMAX = 8;
constexpr int NT_MERGE = 256;              // threads of a merge CTA
constexpr int NCOMB = 4;                 // per-warp states merged at a segment end
constexpr int NSTAGE = 3;
constexpr int BOX_BYTES = 64 * 2 * BLK;       // 64 bf16 columns x 128 rows
constexpr int STAGE_BYTES = 4 * BOX_BYTES;    // K[:, 0:64], K[:, 64:128], V.., V..
constexpr int QSLOT_BYTES = GMAX * HD * 2;
constexpr int SLOT_FLOATS = GMAX * HD + 2 * GMAX;  // partial: O[8][128], m[8], Z[8]
constexpr int MAX_NB = HYLRA_MAX_SEQLEN / BLK;
constexpr int BAR_CONS = 1;     // named barrier of the consumer threads
constexpr int MAX_CTAS = 256;   // grid limit (a merge stages one entry per contributing CTA)
constexpr int MAX_SEGS = 8;     // segments a CTA queues before taking their tickets

// Optional timeline tracing (compile with -DHYLRA_TRACE; off by default and
// then free): per CTA, the producer and the first consumer thread append
// (event code, %globaltimer) pairs to a device buffer set by the host.
#ifdef HYLRA_TRACE
__constant__ unsigned long long* g_hylra_trace = nullptr;  // constant cache: no L2 round trip per event
constexpr int TRACE_PER_CTA = 512;
constexpr int TRACE_CTAS = 256;
__device__ __forceinline__ void trace_event(int& n, int base, int code, int slot) {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  if (g_hylra_trace && n < 255)
    g_hylra_trace[((size_t)slot * TRACE_CTAS + blockIdx.x) * TRACE_PER_CTA + base + n] =
        ((unsigned long long)code << 48) | (t & 0xFFFFFFFFFFFFull);
  ++n;
}
#define HYLRA_TRACE_EV(n, base, code) trace_event(n, base, code, p.trace_slot)
__device__ __forceinline__ void trace_event_cta(int& n, int cta, int code, int slot) {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  if (g_hylra_trace && n < 255 && cta < TRACE_CTAS)
    g_hylra_trace[((size_t)slot * TRACE_CTAS + cta) * TRACE_PER_CTA + n] =
        ((unsigned long long)code << 48) | (t & 0xFFFFFFFFFFFFull);
  ++n;
}
#define HYLRA_TRACE_CTA(n, cta, code) trace_event_cta(n, cta, code, p.trace_slot)
// a raw value (e.g. a cycle count) in place of the timestamp
__device__ __forceinline__ void trace_value_cta(int& n, int cta, int code, int slot,
                                                unsigned long long v) {
  if (g_hylra_trace && n < 255 && cta < TRACE_CTAS)
    g_hylra_trace[((size_t)slot * TRACE_CTAS + cta) * TRACE_PER_CTA + n] =
        ((unsigned long long)code << 48) | (v & 0xFFFFFFFFFFFFull);
  ++n;
}
#define HYLRA_TRACE_VAL(n, cta, code, v) trace_value_cta(n, cta, code, p.trace_slot, v)
#define HYLRA_CLOCK() clock64()
#else
#define HYLRA_TRACE_VAL(n, cta, code, v) ((void)0)
#define HYLRA_CLOCK() 0ll
#define HYLRA_TRACE_CTA(n, cta, code) ((void)0)
#define HYLRA_TRACE_EV(n, base, code) ((void)0)
#endif

struct Params {
  const void* q;
  const void* K;  // read directly by the fp32 kernel
  const void* V;
  const int32_t* seqlens;
  const int64_t* seq_off;
  const int32_t* topk_in;
  float* out;
  int32_t* topk_out;
  uint32_t* status;
  uint32_t* tickets;
  float* partials;
  float* bstat;     // block records, float2 [B*Hkv][r][nbmax] (bstat_at)
  long long cap;    // dense rows per (b, h) plane; 0 = packed layout
  long long total;  // packed rows per KV-head plane
  int B, Hq, Hkv, r, k, max_seqlen, nbmax;
  int idx_wait;      // reuse: topk_in is written by the immediately preceding kernel
  int newest_only;   // block gather: copy only the block holding each sequence's newest token
  int staged;        // reuse: K/V are a staging cache [B][Hkv][k][128][d] whose slot e holds
                     // block topk_in[b][h][e] (written by gather_blocks_kernel)
  int late_from;     // bf16 streaming kernel: CTAs >= late_from start late (their SM is
  int late_deficit;  // still held by the preceding kernel) and take this many units fewer
  int q_wait;        // q and each sequence's newest K/V row come from the preceding kernel
  int upc, nst;      // cluster reuse kernel: blocks per CTA, pipeline stages
  int comb_in_stage; // cluster reuse kernel: the warp states go to stage 0 at the end
  int trace_slot;    // trace builds: which per-launch region of the trace buffer
  float scale_log2;  // log2(e) / sqrt(d)
  long long wait_limit;  // SM clocks after which a bounded wait gives up
};

struct StageMeta {
  int b, h, blk, nvalid, flags, seg_slot, first_slot, ncontrib, nb, pos, pad1, pad2;
};
constexpr int F_SEG_START = 1;
constexpr int F_SEG_END = 2;

// A stage description only ever comes from describe_unit; this re-checks the
// fields that address global memory so that a consumer that gave up waiting
// (HYLRA_STATUS_TIMEOUT) can never write out of bounds.
__device__ __forceinline__ bool meta_sane(const Params& p, const StageMeta& m) {
  const int nslots = (int)gridDim.x + p.B * p.Hkv;
  return m.b >= 0 && m.b < p.B && m.h >= 0 && m.h < p.Hkv && m.blk < p.nbmax && m.nb >= 0 &&
         m.nb <= p.nbmax && m.seg_slot >= 0 && m.seg_slot < nslots && m.first_slot >= 0 &&
         m.ncontrib >= 1 && m.first_slot + m.ncontrib <= nslots && m.nvalid <= BLK;
}

struct alignas(16) SmemCommon {
  alignas(16) float comb_o[NCOMB][GMAX][HD];  // warp states at a segment end; merge/top-k scratch
  float comb_m[NWMAX][GMAX];
  float comb_z[NWMAX][GMAX];
  float mg[GMAX];
  float zg[GMAX];
  float rzg[GMAX];
  float cf[NCOMB][GMAX];  // segment-end scale factors
  int prefix[HYLRA_MAX_BATCH + 1];  // units before sequence b (all heads)
  int hist[256];
  int misc[8];  // 1: radix digit, 2: remaining, 3: list size, 4: abort, 5: digit count
  int warp_sums[NT_MERGE / 32];
  StageMeta segs[MAX_SEGS];  // segments whose partial is stored but not yet ticketed
  int seg_last[MAX_SEGS];
  int nseg;
  int trace_n;    // trace builds: events recorded by consumer thread 0
  int trace_cta;  // trace builds: trace region of this CTA
};
static_assert(sizeof(float) * NCOMB * GMAX * HD >= MAX_NB * 4 + HYLRA_MAX_TOPK * 8,
              "top-k scratch must fit in the combine buffer");
static_assert(sizeof(float) * NCOMB * GMAX * HD >= 2 * MAX_CTAS * GMAX * 4,
              "merge staging must fit in the combine buffer");
static_assert(alignof(SmemCommon) == 16, "top-k reads the combine buffer as uint4");

struct SmemBF16 {
  uint8_t stage[NSTAGE][STAGE_BYTES];  // 1024-byte aligned (128-byte swizzle atoms)
  uint8_t qslot[NSTAGE][QSLOT_BYTES];
  float bst_s[NSTAGE][NW_BF16][GMAX];
  float bst_m[NSTAGE][NW_BF16][GMAX];
  int bst_cnt[NSTAGE];
  StageMeta meta[NSTAGE];
  alignas(8) uint64_t fullK_bar[NSTAGE];  // q rows (segment start) + K tile landed
  alignas(8) uint64_t fullV_bar[NSTAGE];  // V tile landed
  alignas(8) uint64_t empty_bar[NSTAGE];
  SmemCommon c;
};

struct SmemF32 {
  float qs[GMAX][HD];
  float bst_s[2][NW_F32][GMAX];
  float bst_m[2][NW_F32][GMAX];
  SmemCommon c;
};

// ------------------------------------------------------------ work layout

// Sequence length after validation; an invalid length counts as empty.
__device__ __forceinline__ int valid_seqlen(const Params& p, int b, bool report) {
  const int n = p.seqlens[b];
  bool bad = n < 0 || n > p.max_seqlen;
  if (!bad) {
    if (p.cap > 0) {
      bad = (long long)n > p.cap;
    } else {
      const long long o = p.seq_off[b];
      bad = o < 0 || o + n > p.total;
    }
  }
  if (bad) {
    if (report) atomicOr(p.status, HYLRA_STATUS_BAD_SEQLEN);
    return 0;
  }
  return n;
}

__device__ __forceinline__ int units_of(const Params& p, int n, bool full) {
  const int nb = (n + BLK - 1) / BLK;
  return full ? nb : min(p.k, nb);
}

// First row of (b, h) in the 2-D [rows][d] view of K or V.
__device__ __forceinline__ long long row_base(const Params& p, int b, int h) {
  return p.cap > 0 ? ((long long)b * p.Hkv + h) * p.cap : (long long)h * p.total + p.seq_off[b];
}

// Static share of the bf16 streaming kernel: CTA c holds units
// [part_lo(c), part_lo(c+1)).  The CTAs from E on start late (inside a decode
// step their SMs are still held by the preceding kernel while the others
// already stage their first blocks), so each takes D units fewer than the
// rest; D applies only when every late CTA still gets a unit.
__device__ __forceinline__ int late_deficit(const Params& p, long long T, int G) {
  const long long E = min(max(p.late_from, 0), G), L = G - E, D = p.late_deficit;
  return (D > 0 && L > 0 && T + L * D >= (long long)G * (D + 1)) ? (int)D : 0;
}
__device__ __forceinline__ long long part_lo(long long c, long long T, int G, int E, int D) {
  const long long L = G - E;
  return (c * (T + L * D) - (long long)D * G * max(0ll, c - E)) / G;
}
// CTA whose static share holds unit u (binary search over part_lo).
__device__ __forceinline__ int part_owner(long long u, long long T, int G, int E, int D) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (part_lo(mid, T, G, E, D) <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA that owns linear unit u when CTA c holds [floor(c*T/G), floor((c+1)*T/G));
// with G <= T every such range is non-empty.
__device__ __forceinline__ int owner_cta(long long u, long long T, int G) {
  return (int)(((u + 1) * G - 1) / T);
}

// Block records (max, probability sum) of reset layers: float2 at
// [b * Hkv + h][g][block], head-major so that consecutive blocks of one head
// are adjacent (the merge reads them one block per lane).
__device__ __forceinline__ size_t bstat_at(const Params& p, int bh, int g, int beta) {
  return (((size_t)bh * p.r + g) * p.nbmax + beta) * 2;
}

// prefix[b] = number of units of sequences 0..b-1 (all KV heads); warp 0.
__device__ void build_prefix(const Params& p, SmemCommon& c, bool full) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const int per = (p.B + 31) / 32;
  const int b0 = min(p.B, lane * per), b1 = min(p.B, b0 + per);
  int local = 0;
  for (int b = b0; b < b1; ++b)
    local += units_of(p, valid_seqlen(p, b, blockIdx.x == 0), full) * p.Hkv;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - local;
  for (int b = b0; b < b1; ++b) {
    c.prefix[b] = run;
    run += units_of(p, valid_seqlen(p, b, false), full) * p.Hkv;
  }
  if (lane == 31) c.prefix[p.B] = incl;
}

// Sequences without units still need an output: zeros (and -1 indices).
template <bool FULL>
__device__ void write_empty_outputs(const Params& p, const SmemCommon& c) {
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    if (c.prefix[b + 1] != c.prefix[b]) continue;
    griddep_wait();  // outputs may be buffers the preceding kernel writes
    float* o = p.out + (size_t)b * p.Hq * HD;
    for (int i = threadIdx.x; i < p.Hq * HD; i += blockDim.x) o[i] = 0.f;
    if (FULL) {
      int32_t* t = p.topk_out + (size_t)b * p.Hkv * p.k;
      for (int i = threadIdx.x; i < p.Hkv * p.k; i += blockDim.x) t[i] = -1;
    }
  }
}

// Walks units (b, h, j) in linear order.
struct UnitIter {
  int b, h, j, U;
  __device__ void seek(const SmemCommon& c, const Params& p, int u) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (c.prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    b = lo;
    U = (c.prefix[b + 1] - c.prefix[b]) / p.Hkv;
    const int off = u - c.prefix[b];
    h = off / U;
    j = off - h * U;
  }
  __device__ void advance(const SmemCommon& c, const Params& p) {
    if (++j < U) return;
    j = 0;
    if (++h < p.Hkv) return;
    h = 0;
    do { ++b; } while (b < p.B && c.prefix[b + 1] == c.prefix[b]);
    if (b < p.B) U = (c.prefix[b + 1] - c.prefix[b]) / p.Hkv;
  }
};

// Everything a unit needs besides its data.  seqlen: the validated length of
// sequence it.b; blk_raw: the unit's block (FULL) or its reused index entry.
template <bool FULL>
__device__ __forceinline__ StageMeta describe_unit(const Params& p, const SmemCommon& c,
                                                   const UnitIter& it, int i, int n, int T,
                                                   int G, int seqlen, int blk_raw, bool report) {
  StageMeta m;
  const int bh = it.b * p.Hkv + it.h;
  const int nb = (seqlen + BLK - 1) / BLK;
  int blk = blk_raw;
  if (!FULL && (blk < 0 || blk >= nb)) {
    if (blk != -1 && report) atomicOr(p.status, HYLRA_STATUS_BAD_INDEX);
    blk = -1;
  }
  const int start = c.prefix[it.b] + it.h * it.U;
  const int cf = owner_cta(start, T, G);
  const int cl = owner_cta((long long)start + it.U - 1, T, G);
  m.b = it.b;
  m.h = it.h;
  m.blk = blk;
  m.nvalid = blk >= 0 ? min(BLK, seqlen - blk * BLK) : 0;
  m.flags = ((i == 0 || it.j == 0) ? F_SEG_START : 0) | ((i == n - 1 || it.j == it.U - 1) ? F_SEG_END : 0);
  m.seg_slot = (int)blockIdx.x + bh;
  m.first_slot = cf + bh;
  m.ncontrib = cl - cf + 1;
  m.nb = nb;
  m.pos = it.j;  // place in the (b, h) index list (reuse) or block (reset)
  m.pad1 = m.pad2 = 0;
  return m;
}

__device__ __forceinline__ int unit_index_entry(const Params& p, const UnitIter& it) {
  return __ldcg(p.topk_in + ((size_t)it.b * p.Hkv + it.h) * p.k + it.j);
}

// ------------------------------------------------------------------ top-k

// Top-k of the block scores keys[0..nb) (fp32 bit patterns of non-negative
// scores, so unsigned order is numeric order): rank order, score descending,
// lower block index first among equal scores; slots k'..k-1 get -1.
// Called by the NT merge threads (ct = 0..NT-1).
//
// A key "beats" another when it is larger, or equal with a lower index; the
// answer is the kp keys beaten by fewer than kp others.  Up to NT keys and
// kp <= 32: per-warp sorted lists ranked by counting (below).  Other cases
// with kp <= 32: a merge tree of per-warp sorted lists (topk_tree).  Larger
// kp: a radix select on the keys' bit patterns.

// Warp-level compare-exchange networks on 64-bit values, descending.  A
// warp holds 32 * N values, element e = lane * N + i in register i: pairs at
// distance j < N are in one lane's registers, the others one shuffle apart.
template <int N>
__device__ __forceinline__ void cx_desc(uint64_t (&v)[N], int lane, int j, int k) {
  if (j < N) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if (i & j) continue;
      // (lane, i) is the lower element of its pair; its run of k elements
      // is sorted descending when bit k of its index is clear
      const bool desc = ((lane * N + i) & k) == 0;
      const uint64_t a = v[i], b = v[i | j];
      const bool swap = desc ? (a < b) : (a > b);
      v[i] = swap ? b : a;
      v[i | j] = swap ? a : b;
    }
  } else {
    const int lj = j / N;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, v[i], lj);
      const bool desc = ((lane * N + i) & k) == 0;
      const bool lower = (lane & lj) == 0;
      v[i] = (lower == desc) ? (v[i] > o ? v[i] : o) : (v[i] < o ? v[i] : o);
    }
  }
}

// Sorts a bitonic sequence of 32 * N values descending (one merge pass).
template <int N>
__device__ __forceinline__ void warp_bitonic_merge_desc(uint64_t (&v)[N], int lane) {
#pragma unroll
  for (int j = 16 * N; j > 0; j >>= 1) cx_desc<N>(v, lane, j, 64 * N);  // bit 64N: never set
}

// Top-k' for k' <= LIST = 32 * LPL, without data-dependent work.  (key,
// block) pairs compare as distinct 64-bit composites (score descending, block
// ascending).  Two facts do all the work: for A and B sorted descending,
// max(A[e], B[LIST-1-e]) is bitonic and holds the LIST largest of A and B
// (so one merge pass sorts them), and the largest of a union are the
// largest of the parts' largest.  Each warp keeps a sorted list of its
// LIST largest so far; per round of 32 keys (one per lane) it sorts them
// and merges them in.  Then the warps' lists merge pairwise in a tree.
// The networks run inside loops, not unrolled, so the code that runs once
// per launch stays small (it is fetched cold).
template <int NT, int LPL, int BAR>
__device__ void topk_tree(const uint32_t* keys, uint32_t* scratch, int32_t* dst, int nb, int kp,
                          int k, int ct) {
  constexpr int NW = NT / 32, LIST = 32 * LPL;
  static_assert((NW & (NW - 1)) == 0, "power-of-two warps");
  static_assert((MAX_NB + 256) * 4 + NW * LIST * 8 <= NCOMB * GMAX * HD * 4,
                "keys, maxima and lists share the combine area");
  uint64_t* lists = reinterpret_cast<uint64_t*>(scratch + 256);  // [NW][LIST]
  const int lane = ct & 31, wid = ct >> 5;
  for (int slot = kp + ct; slot < k; slot += NT) dst[slot] = -1;
  uint64_t L[LPL];
#pragma unroll
  for (int i = 0; i < LPL; ++i) L[i] = 0ull;
#pragma unroll 1
  for (int base = wid * 32; base < nb; base += NT) {
    const int beta = base + lane;
    uint64_t x[1] = {beta < nb ? ((uint64_t)keys[beta] << 32) | (uint32_t)~(uint32_t)beta : 0ull};
    // nothing to do when no key beats the list's last entry
    const uint64_t last = __shfl_sync(0xffffffffu, L[LPL - 1], 31);
    if (!__any_sync(0xffffffffu, x[0] > last)) continue;
#pragma unroll
    for (int kk = 2; kk <= 32; kk <<= 1)
#pragma unroll
      for (int j = kk >> 1; j > 0; j >>= 1) cx_desc<1>(x, lane, j, kk);
    // the 32 sorted keys, padded with zeros to LIST, reversed against L
#pragma unroll
    for (int i = 0; i < LPL; ++i) {
      const int f = LIST - 1 - (lane * LPL + i);
      const uint64_t xf = __shfl_sync(0xffffffffu, x[0], f & 31);
      const uint64_t b = f < 32 ? xf : 0ull;
      L[i] = L[i] > b ? L[i] : b;
    }
    warp_bitonic_merge_desc<LPL>(L, lane);
  }
#pragma unroll
  for (int i = 0; i < LPL; ++i) lists[wid * LIST + lane * LPL + i] = L[i];
  named_bar_sync(BAR, NT);
  // Every warp takes every level's barrier (the same barrier at the same
  // count as the caller's, which the early warps may reach next).
#pragma unroll 1
  for (int span = 1; span < NW; span <<= 1) {
    const int nm = NW / (2 * span);  // merging warps at this level
    if (wid < nm) {
      const uint64_t* A = lists + (2 * span * wid) * LIST;
      const uint64_t* B = A + span * LIST;
#pragma unroll
      for (int i = 0; i < LPL; ++i) {
        const int e = lane * LPL + i;
        const uint64_t a = A[e], b = B[LIST - 1 - e];
        L[i] = a > b ? a : b;
      }
      warp_bitonic_merge_desc<LPL>(L, lane);
      if (nm > 1) {
        __syncwarp();
#pragma unroll
        for (int i = 0; i < LPL; ++i) lists[(2 * span * wid) * LIST + lane * LPL + i] = L[i];
      }
    }
    if (nm > 1) named_bar_sync(BAR, NT);
  }
  if (wid != 0) return;
  // warp 0 holds the answer (with one warp, its own list)
#pragma unroll
  for (int i = 0; i < LPL; ++i) {
    const int e = lane * LPL + i;
    if (e < kp) dst[e] = (int32_t)~(uint32_t)(L[i] & 0xffffffffull);
  }
}

template <int NT, int BAR = BAR_CONS>
__device__ void topk_select(const Params& p, SmemCommon& c, int bh, int nb, int ct) {
  constexpr int NW = NT / 32;
  uint32_t* keys = reinterpret_cast<uint32_t*>(&c.comb_o[0][0][0]);
  uint32_t* tmax = keys + MAX_NB;  // scratch past the keys (lists)
  int32_t* dst = p.topk_out + (size_t)bh * p.k;
  const int kp = min(p.k, nb);
  const int lane = ct & 31, wid = ct >> 5;

  if (nb <= NT && kp <= 32) {
    // One key per thread.  (key, block) pairs compare as one 64-bit
    // composite, descending by key then ascending by block, so all are
    // distinct.  Each warp places its 32 composites in sorted order (an
    // entry's place = how many of the warp's composites exceed it) and keeps
    // the first kp.  An entry's global rank is the sum over warps of how many
    // of their kept entries exceed it (a binary search in each sorted list);
    // the entries of rank < kp are the answer.
    uint64_t* comp = reinterpret_cast<uint64_t*>(tmax + 256);  // [NT] composites
    uint64_t* lists = comp + NT;                                 // [NW][32] sorted
    const uint64_t v = ct < nb ? ((uint64_t)keys[ct] << 32) | (uint32_t)~(uint32_t)ct : 0ull;
    comp[ct] = v;
    lists[ct] = 0ull;  // lists cover NW * 32 == NT entries; unused places stay 0
    named_bar_sync(BAR, NT);
    // place within the warp: how many of its 32 composites exceed v
    int rw = 0;
    const ulonglong2* wc = reinterpret_cast<const ulonglong2*>(comp + wid * 32);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const ulonglong2 o = wc[j];
      rw += (o.x > v) + (o.y > v);
    }
    if (rw < kp) lists[wid * 32 + rw] = v;
    named_bar_sync(BAR, NT);
    if (rw < kp && v != 0ull) {
      // how many entries of each list exceed v: a binary search over the 32
      // places (a list past its kp entries holds zeros, below every key), the
      // NW searches in lock step, each step a select (independent loads in
      // flight, no branch); in its own warp's list an entry finds exactly
      // `rw` predecessors
      int pos[NW];
#pragma unroll
      for (int w = 0; w < NW; ++w) pos[w] = 0;
#pragma unroll
      for (int step = 16; step > 0; step >>= 1) {
#pragma unroll
        for (int w = 0; w < NW; ++w)
          pos[w] += lists[w * 32 + pos[w] + step - 1] > v ? step : 0;
      }
#pragma unroll
      for (int w = 0; w < NW; ++w) pos[w] += lists[w * 32 + pos[w]] > v ? 1 : 0;
      int rank = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) rank += pos[w];
      if (rank < kp) dst[rank] = (int32_t)~(uint32_t)(v & 0xffffffffull);
    }
    for (int slot = kp + ct; slot < p.k; slot += NT) dst[slot] = -1;
    return;
  }

  if (kp <= 32) {
    topk_tree<NT, 1, BAR>(keys, tmax, dst, nb, kp, p.k, ct);
    return;
  }

  // Radix select of the kp-th largest key, 8 bits per pass.  A pass whose
  // chosen digit holds exactly the `remain` keys still wanted ends the
  // search: every key whose bits above `shift` reach the prefix is taken.
  uint32_t prefix = 0;
  int remain = kp;
  int shift = 0;
  bool whole = false;  // the last digit's keys are all taken
  for (int pass = 0; pass < 4 && !whole; ++pass) {
    shift = 24 - 8 * pass;
    for (int i = ct; i < 256; i += NT) c.hist[i] = 0;
    if (ct == 0) c.misc[3] = 0;
    named_bar_sync(BAR, NT);
    // one shared atomic per distinct digit per warp (scores of one head
    // mostly share their top bits, so per-thread atomics would serialize)
    for (int beta0 = 0; beta0 < nb; beta0 += NT) {
      const int beta = beta0 + ct;
      const uint32_t key = beta < nb ? keys[beta] : 0u;
      const bool match = beta < nb && (pass == 0 || ((key ^ prefix) >> (shift + 8)) == 0u);
      const uint32_t digit = match ? ((key >> shift) & 255u) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (match && (__ffs(peers) - 1) == lane) atomicAdd(&c.hist[digit], __popc(peers));
    }
    named_bar_sync(BAR, NT);
    if (wid == 0) {
      int cnt[8];
      int local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = c.hist[255 - 8 * lane - i];
        local += cnt[i];
      }
      int incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int excl = incl - local;
      if (excl < remain && remain <= incl) {
        int acc = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc + cnt[i] >= remain) {
            c.misc[1] = 255 - 8 * lane - i;
            c.misc[2] = remain - acc;
            c.misc[5] = cnt[i];  // keys with this digit
            break;
          }
          acc += cnt[i];
        }
      }
    }
    named_bar_sync(BAR, NT);
    prefix |= (uint32_t)c.misc[1] << shift;
    remain = c.misc[2];
    whole = c.misc[5] == remain;
  }
  // tau: the kp-th largest key's bits from `shift` up.  Keep every key whose
  // bits from `shift` up exceed tau's, and of those equal to it all of them
  // (whole digit) or the lowest-index `remain` (ties after the last pass).
  const uint32_t tau = prefix >> shift;

  uint2* rlist = reinterpret_cast<uint2*>(keys + MAX_NB);
  const int per = (nb + NT - 1) / NT;
  const int b0 = min(nb, ct * per), b1 = min(nb, b0 + per);
  int eq = 0;
  for (int beta = b0; beta < b1; ++beta) eq += (keys[beta] >> shift) == tau;
  int incl = eq;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) c.warp_sums[wid] = incl;
  named_bar_sync(BAR, NT);
  int before = incl - eq;
#pragma unroll
  for (int w = 0; w < NW; ++w)
    if (w < wid) before += c.warp_sums[w];
  for (int beta = b0; beta < b1; ++beta) {
    const uint32_t key = keys[beta];
    bool sel = (key >> shift) > tau;
    if ((key >> shift) == tau) {
      sel = whole || before < remain;
      ++before;
    }
    if (sel) {
      const int pos = atomicAdd(&c.misc[3], 1);
      if (pos < kp) rlist[pos] = make_uint2(key, (uint32_t)beta);  // exactly kp are selected
    }
  }
  named_bar_sync(BAR, NT);
  for (int e = ct; e < kp; e += NT) {
    const uint2 me = rlist[e];
    int rank = 0;
    for (int j = 0; j < kp; ++j) {
      const uint2 o = rlist[j];
      rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
    }
    dst[rank] = (int32_t)me.y;
  }
  for (int slot = kp + ct; slot < p.k; slot += NT) dst[slot] = -1;
}

// ---------------------------------------------------------------- merging

// The last CTA of (b, h): LSE-merge every contributor's partial into out;
// on reset layers also score the blocks and select the top-k.  The merge
// sits on the kernel's tail, so it is one L2 round trip: every thread loads
// the (max, sum, row) of its contributors together and merges them online;
// the NT threads split into G groups over the contributors, combined once
// through shared memory.
template <bool FULL, int NT>
__device__ void merge_bh(const Params& p, SmemCommon& c, const StageMeta& m, int ct) {
  constexpr int CB = NT >= 512 ? 6 : 10;  // contributors per thread and batch of loads
  const int bh = m.b * p.Hkv + m.h;
  const int nc = m.ncontrib;
  const int r = p.r;
  const float* pbase = p.partials + (size_t)m.first_slot * SLOT_FLOATS;
  const int kp = min(p.k, m.nb);
  const int32_t* idx = p.topk_in + (size_t)bh * p.k;
  const int32_t my_idx = (!FULL && ct < kp) ? __ldcg(idx + ct) : -1;
  // block records of the first block of this thread (reset layers)
  float2 sv0[GMAX];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    sv0[g] = make_float2(0.f, -INFINITY);
    if (FULL && ct < m.nb && g < r)
      sv0[g] = __ldcg(reinterpret_cast<const float2*>(
          p.bstat + bstat_at(p, bh, g, ct)));
  }

  const int ncol = r * (HD / 4);             // float4 output columns
  const int G = ncol >= NT ? 1 : min(NWMAX, NT / ncol);  // contributor groups
  float4* red = reinterpret_cast<float4*>(&c.comb_o[0][0][0]);  // [G][ncol]
  for (int t = ct; t < G * ncol; t += NT) {
    const int q = t / ncol, col = t - q * ncol;
    const int g = col / (HD / 4), d4 = col - g * (HD / 4);
    float M = -INFINITY, Z = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = q; j0 < nc; j0 += G * CB) {
      float mv[CB], zv[CB];
      float4 ov[CB];
#pragma unroll
      for (int u = 0; u < CB; ++u) {
        const int j = j0 + u * G;
        mv[u] = -INFINITY;
        if (j < nc) {
          const float* sl = pbase + (size_t)j * SLOT_FLOATS;
          mv[u] = __ldcg(sl + GMAX * HD + g);
          zv[u] = __ldcg(sl + GMAX * HD + GMAX + g);
          ov[u] = __ldcg(reinterpret_cast<const float4*>(sl + g * HD + 4 * d4));
        }
      }
#pragma unroll
      for (int u = 0; u < CB; ++u) {
        if (mv[u] == -INFINITY) continue;
        if (mv[u] > M) {
          const float f = M == -INFINITY ? 0.f : ex2_approx(M - mv[u]);
          acc.x *= f;
          acc.y *= f;
          acc.z *= f;
          acc.w *= f;
          Z *= f;
          M = mv[u];
        }
        const float f = ex2_approx(mv[u] - M);
        acc.x = fmaf(ov[u].x, f, acc.x);
        acc.y = fmaf(ov[u].y, f, acc.y);
        acc.z = fmaf(ov[u].z, f, acc.z);
        acc.w = fmaf(ov[u].w, f, acc.w);
        Z = fmaf(zv[u], f, Z);
      }
    }
    red[t] = acc;
    if (d4 == 0) {
      c.comb_m[q][g] = M;
      c.comb_z[q][g] = Z;
    }
  }
  if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 16 << 8);
  named_bar_sync(BAR_CONS, NT);
  for (int col = ct; col < ncol; col += NT) {
    const int g = col / (HD / 4), d4 = col - g * (HD / 4);
    float M = -INFINITY;
    for (int q = 0; q < G; ++q) M = fmaxf(M, c.comb_m[q][g]);
    float Z = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int q = 0; q < G; ++q) {
        const float mq = c.comb_m[q][g];
        if (mq == -INFINITY) continue;
        const float f = ex2_approx(mq - M);
        const float4 v = red[q * ncol + col];
        acc.x = fmaf(v.x, f, acc.x);
        acc.y = fmaf(v.y, f, acc.y);
        acc.z = fmaf(v.z, f, acc.z);
        acc.w = fmaf(v.w, f, acc.w);
        Z = fmaf(c.comb_z[q][g], f, Z);
      }
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (Z > 0.f) o = make_float4(acc.x / Z, acc.y / Z, acc.z / Z, acc.w / Z);
    *reinterpret_cast<float4*>(p.out + ((size_t)m.b * p.Hq + (size_t)m.h * r + g) * HD + 4 * d4) = o;
    if (d4 == 0) {
      c.mg[g] = M;
      c.zg[g] = Z;
      c.rzg[g] = Z > 0.f ? 1.f / Z : 0.f;
    }
  }
  if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 17 << 8);
  if (FULL) {
    named_bar_sync(BAR_CONS, NT);  // head maxima and sums visible; comb_o free
    uint32_t* keys = reinterpret_cast<uint32_t*>(&c.comb_o[0][0][0]);
    bool nonfinite = false;
    for (int beta = ct; beta < m.nb; beta += NT) {
      float2 sv[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (beta == ct) {
          sv[g] = sv0[g];
        } else {
          sv[g] = g < r ? __ldcg(reinterpret_cast<const float2*>(
                              p.bstat + bstat_at(p, bh, g, beta)))
                        : make_float2(0.f, -INFINITY);
        }
      }
      float score = 0.f;
#pragma unroll
      for (int g = 0; g < GMAX; ++g)
        if (g < r && c.zg[g] > 0.f && sv[g].y != -INFINITY)
          score += sv[g].x * exp2f(sv[g].y - c.mg[g]) * c.rzg[g];
      uint32_t key = 0u;
      if (isfinite(score)) {
        if (score > 0.f) key = __float_as_uint(score);
      } else {
        nonfinite = true;
      }
      keys[beta] = key;
    }
    if (nonfinite) atomicOr(p.status, HYLRA_STATUS_NONFINITE);
    named_bar_sync(BAR_CONS, NT);
    if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 12 << 8);
    topk_select<NT>(p, c, bh, m.nb, ct);
    if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 13 << 8);
  } else {
    // a reused list naming one block twice counts that block twice: flag it
    named_bar_sync(BAR_CONS, NT);  // comb_o free
    int32_t* sidx = reinterpret_cast<int32_t*>(&c.comb_o[0][0][0]);
    for (int e = ct; e < kp; e += NT) sidx[e] = e == ct ? my_idx : __ldcg(idx + e);
    named_bar_sync(BAR_CONS, NT);
    bool dup = false;
    for (int e = ct; e < kp; e += NT) {
      const int32_t v = sidx[e];
      if (v < 0) continue;
      for (int j = 0; j < e; ++j) dup |= sidx[j] == v;
    }
    if (dup) atomicOr(p.status, HYLRA_STATUS_DUP_INDEX);
  }
  if (ct == 0) p.tickets[bh] = 0u;  // ready for the next launch
  named_bar_sync(BAR_CONS, NT);
}

// Segment end: comb_*[0..NCOMB) hold partial states (m, Z, O) of this CTA's
// share of (b, h).  Merge them and store the CTA's partial (no fence: the
// ticket that makes it visible is taken later, in flush_segments), and queue
// the segment.  Ends with a barrier (comb_* may be rewritten afterwards).
template <int NT, bool QUEUE>
__device__ void store_partial(const Params& p, SmemCommon& c, const StageMeta& m, int ct) {
  const bool sane = meta_sane(p, m);
  float* slot = p.partials + (size_t)(sane ? m.seg_slot : 0) * SLOT_FLOATS;
  if (sane && ct < p.r) {
    const int g = ct;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NCOMB; ++w) M = fmaxf(M, c.comb_m[w][g]);
    float Z = 0.f;
#pragma unroll
    for (int w = 0; w < NCOMB; ++w) {
      const float mw = c.comb_m[w][g];
      const float f = (M == -INFINITY || mw == -INFINITY) ? 0.f : exp2f(mw - M);
      c.cf[w][g] = f;
      Z += c.comb_z[w][g] * f;
    }
    slot[GMAX * HD + g] = M;
    slot[GMAX * HD + GMAX + g] = Z;
  }
  named_bar_sync(BAR_CONS, NT);
  if (sane) {
    for (int pr = ct; pr < p.r * HD; pr += NT) {
      const int g = pr / HD, d = pr - g * HD;
      float O = 0.f;
#pragma unroll
      for (int w = 0; w < NCOMB; ++w) O = fmaf(c.comb_o[w][g][d], c.cf[w][g], O);
      slot[g * HD + d] = O;
    }
    if (QUEUE && ct == 0) c.segs[c.nseg++] = m;
  }
  named_bar_sync(BAR_CONS, NT);
}

// Make this CTA's stored partials visible, take one ticket per queued
// segment, and merge every (b, h) this CTA finished last.
template <bool FULL, int NT>
__device__ void flush_segments(const Params& p, SmemCommon& c, int ct) {
  __threadfence();
  named_bar_sync(BAR_CONS, NT);
  if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 14 << 8);
  const int ns = c.nseg;
  if (ct < ns) {
    const StageMeta& m = c.segs[ct];
    const uint32_t old = atomic_add_acq_rel_gpu(p.tickets + m.b * p.Hkv + m.h, 1u);
    c.seg_last[ct] = (old == (uint32_t)(m.ncontrib - 1)) ? 1 : 0;
  }
  named_bar_sync(BAR_CONS, NT);
  if (ct == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 15 << 8);
  for (int k = 0; k < ns; ++k) {
    if (c.seg_last[k]) {
      __threadfence();
      const StageMeta m = c.segs[k];
      merge_bh<FULL, NT>(p, c, m, ct);
    }
  }
  if (ct == 0) c.nseg = 0;
  named_bar_sync(BAR_CONS, NT);
}

// Block record of one head g from the nw warps' shares of a block: the
// block's own max and its probability sum relative to that max.
template <int NW>
__device__ __forceinline__ void combine_block_record(const float (*bs)[GMAX],
                                                     const float (*bm)[GMAX], int g, float* dst) {
  float mm = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) mm = fmaxf(mm, bm[w][g]);
  float ss = 0.f;
  if (mm != -INFINITY) {
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = bm[w][g];
      if (mw != -INFINITY) ss += bs[w][g] * exp2f(mw - mm);
    }
  }
  dst[0] = ss;
  dst[1] = mm;
}

// ------------------------------------------------------ consumer warp state

// Online-softmax attention state of one consumer warp of the bf16 kernels:
// tokens 16*cw .. 16*cw+15 of every block, the r <= 8 q-heads of one KV head.
// The fragments follow the mma.sync m16n8k16 layouts: this lane holds heads
// 2*c4 (A) and 2*c4+1 (B), tokens g4 and g4+8 of S^T, and O^T rows
// (d = 16*dm + g4 [+8]) for those two heads.
struct WarpAttn {
  float o[8][4];
  float m_run[2], z_run[2];
  uint32_t qf[8][2];
  int lane, g4, c4, tokw, krow, kchi, vrow, vchi, xr;

  __device__ __forceinline__ void init(int cw, int lane_) {
    lane = lane_;
    g4 = lane >> 2;
    c4 = lane & 3;
    tokw = cw * 16;
    const int mi = lane >> 3;
    // this lane's ldmatrix rows: K (non-transposed) and V (transposed) tiles
    krow = tokw + (lane & 7) + (mi & 1) * 8;
    kchi = mi >> 1;
    vrow = tokw + (lane & 7) + (mi >> 1) * 8;
    vchi = mi & 1;
    xr = lane & 7;  // == krow & 7 == vrow & 7
    reset();
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) qf[kt][0] = qf[kt][1] = 0u;
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int dm = 0; dm < 8; ++dm)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[dm][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    z_run[0] = z_run[1] = 0.f;
  }

  // q rows [r][128] bf16 in shared memory -> B operand of S^T = K Q^T
  __device__ __forceinline__ void load_q(const uint8_t* qrows, int r) {
    const uint32_t* qs = reinterpret_cast<const uint32_t*>(qrows);
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      qf[kt][0] = g4 < r ? qs[(g4 * HD + kt * 16 + 2 * c4) >> 1] : 0u;
      qf[kt][1] = g4 < r ? qs[(g4 * HD + kt * 16 + 8 + 2 * c4) >> 1] : 0u;
    }
  }

  // One 128-token block in a stage (K at stage, V at stage + 2 boxes).  Waits
  // for V itself.  Returns the block-local max and probability sum (relative
  // to that max) of this warp's tokens for heads A and B.
  __device__ __forceinline__ void block(uint8_t* stage, int nvalid, float scale_log2,
                                        uint64_t* fullV, uint32_t ph, volatile int* abort_flag,
                                        long long lim, float& mxA, float& mxB, float& sA,
                                        float& sB) {
    const uint32_t kbase = smem_u32(stage);
    const uint32_t vbase = kbase + 2 * BOX_BYTES;
    const bool partial = nvalid < BLK;
    float x[4];
    {  // S^T = K Q^T for this warp's 16 tokens, two accumulation chains
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kb = kbase + krow * 128;
#pragma unroll
      for (int kt = 0; kt < 8; ++kt) {
        const int ch = 2 * kt + kchi;
        const uint32_t addr = kb + (ch >> 3) * BOX_BYTES + (((ch & 7) ^ xr) << 4);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(addr, r0, r1, r2, r3);
        mma_bf16_16816((kt & 1) ? a1 : a0, r0, r1, r2, r3, qf[kt][0], qf[kt][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = (a0[e] + a1[e]) * scale_log2;
        if (partial) {
          const int tok = tokw + g4 + ((e & 2) ? 8 : 0);
          if (tok >= nvalid) v = -INFINITY;
        }
        x[e] = v;
      }
    }
    mbar_wait_bounded(fullV, ph, abort_flag, lim);
    if (partial) {
      // rows past the sequence end may hold anything (even NaN): zero V
      for (int idx = lane; idx < 16 * 16; idx += 32) {
        const int row = tokw + (idx >> 4);
        if (row < nvalid) continue;
        const int ch = idx & 15;
        uint8_t* ptr = stage + 2 * BOX_BYTES + (ch >> 3) * BOX_BYTES + row * 128 + (ch & 7) * 16;
        *reinterpret_cast<uint4*>(ptr) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    // block-local max and sums for heads A and B
    mxA = fmaxf(x[0], x[2]);
    mxB = fmaxf(x[1], x[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, off));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, off));
    }
    const float msA = mxA == -INFINITY ? 0.f : mxA;
    const float msB = mxB == -INFINITY ? 0.f : mxB;
    const float p0 = ex2_approx(x[0] - msA), p1 = ex2_approx(x[1] - msB);
    const float p2 = ex2_approx(x[2] - msA), p3 = ex2_approx(x[3] - msB);
    sA = p0 + p2;
    sB = p1 + p3;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, off);
      sB += __shfl_xor_sync(0xffffffffu, sB, off);
    }
    // online softmax update (rescale only when a running max moved)
    const float mnA = fmaxf(m_run[0], mxA), mnB = fmaxf(m_run[1], mxB);
    float alA = 1.f, beA = 0.f, alB = 1.f, beB = 0.f;
    if (mnA != -INFINITY) {
      alA = ex2_approx(m_run[0] - mnA);
      beA = ex2_approx(mxA - mnA);
    }
    if (mnB != -INFINITY) {
      alB = ex2_approx(m_run[1] - mnB);
      beB = ex2_approx(mxB - mnB);
    }
    z_run[0] = z_run[0] * alA + sA * beA;
    z_run[1] = z_run[1] * alB + sB * beB;
    m_run[0] = mnA;
    m_run[1] = mnB;
    if (__any_sync(0xffffffffu, alA != 1.f || alB != 1.f)) {
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        o[dm][0] *= alA;
        o[dm][1] *= alB;
        o[dm][2] *= alA;
        o[dm][3] *= alB;
      }
    }
    // P^T to the B-operand layout, then O^T += V^T P^T
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0 * beA, p1 * beB));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2 * beA, p3 * beB));
    const uint32_t vb = vbase + vrow * 128;
#pragma unroll
    for (int dm = 0; dm < 8; ++dm) {
      const int ch = 2 * dm + vchi;
      const uint32_t addr = vb + (ch >> 3) * BOX_BYTES + (((ch & 7) ^ xr) << 4);
      uint32_t r0, r1, r2, r3;
      ldsm_x4_trans(addr, r0, r1, r2, r3);
      mma_bf16_16816(o[dm], r0, r1, r2, r3, pb0, pb1);
    }
  }

  // Zero the V rows of a partial block past the sequence end (they may hold
  // anything, even NaN) before the PV step reads them.
  __device__ __forceinline__ void zero_tail_v(uint8_t* stage, int nvalid) {
    for (int idx = lane; idx < 16 * 16; idx += 32) {
      const int row = tokw + (idx >> 4);
      if (row < nvalid) continue;
      const int ch = idx & 15;
      uint8_t* ptr = stage + 2 * BOX_BYTES + (ch >> 3) * BOX_BYTES + row * 128 + (ch & 7) * 16;
      *reinterpret_cast<uint4*>(ptr) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    __syncwarp();
  }

  // Two staged blocks as one 256-token step (reuse layers): the two QK
  // chains, one softmax update and the two PV chains interleave, so the
  // pair costs little more than one block.
  __device__ __forceinline__ void block2(uint8_t* st0, int nv0, uint64_t* fullV0, uint32_t ph0,
                                         uint8_t* st1, int nv1, uint64_t* fullV1, uint32_t ph1,
                                         float scale_log2, volatile int* abort_flag, long long lim) {
    float x0[4], x1[4];
    {
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      float b0[4] = {0.f, 0.f, 0.f, 0.f}, b1[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kb0 = smem_u32(st0) + krow * 128, kb1 = smem_u32(st1) + krow * 128;
#pragma unroll
      for (int kt = 0; kt < 8; ++kt) {
        const int ch = 2 * kt + kchi;
        const uint32_t off = (ch >> 3) * BOX_BYTES + (((ch & 7) ^ xr) << 4);
        uint32_t r0, r1, r2, r3, t0, t1, t2, t3;
        ldsm_x4(kb0 + off, r0, r1, r2, r3);
        ldsm_x4(kb1 + off, t0, t1, t2, t3);
        mma_bf16_16816((kt & 1) ? a1 : a0, r0, r1, r2, r3, qf[kt][0], qf[kt][1]);
        mma_bf16_16816((kt & 1) ? b1 : b0, t0, t1, t2, t3, qf[kt][0], qf[kt][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tokw + g4 + ((e & 2) ? 8 : 0);
        x0[e] = tok < nv0 ? (a0[e] + a1[e]) * scale_log2 : -INFINITY;
        x1[e] = tok < nv1 ? (b0[e] + b1[e]) * scale_log2 : -INFINITY;
      }
    }
    mbar_wait_bounded(fullV0, ph0, abort_flag, lim);
    mbar_wait_bounded(fullV1, ph1, abort_flag, lim);
    if (nv0 < BLK) zero_tail_v(st0, nv0);
    if (nv1 < BLK) zero_tail_v(st1, nv1);
    // max and sums over the pair's tokens for heads A and B
    float mxA = fmaxf(fmaxf(x0[0], x0[2]), fmaxf(x1[0], x1[2]));
    float mxB = fmaxf(fmaxf(x0[1], x0[3]), fmaxf(x1[1], x1[3]));
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, off));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, off));
    }
    const float msA = mxA == -INFINITY ? 0.f : mxA;
    const float msB = mxB == -INFINITY ? 0.f : mxB;
    const float p00 = ex2_approx(x0[0] - msA), p01 = ex2_approx(x0[1] - msB);
    const float p02 = ex2_approx(x0[2] - msA), p03 = ex2_approx(x0[3] - msB);
    const float p10 = ex2_approx(x1[0] - msA), p11 = ex2_approx(x1[1] - msB);
    const float p12 = ex2_approx(x1[2] - msA), p13 = ex2_approx(x1[3] - msB);
    float sA = (p00 + p02) + (p10 + p12);
    float sB = (p01 + p03) + (p11 + p13);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, off);
      sB += __shfl_xor_sync(0xffffffffu, sB, off);
    }
    const float mnA = fmaxf(m_run[0], mxA), mnB = fmaxf(m_run[1], mxB);
    float alA = 1.f, beA = 0.f, alB = 1.f, beB = 0.f;
    if (mnA != -INFINITY) {
      alA = ex2_approx(m_run[0] - mnA);
      beA = ex2_approx(mxA - mnA);
    }
    if (mnB != -INFINITY) {
      alB = ex2_approx(m_run[1] - mnB);
      beB = ex2_approx(mxB - mnB);
    }
    z_run[0] = z_run[0] * alA + sA * beA;
    z_run[1] = z_run[1] * alB + sB * beB;
    m_run[0] = mnA;
    m_run[1] = mnB;
    if (__any_sync(0xffffffffu, alA != 1.f || alB != 1.f)) {
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        o[dm][0] *= alA;
        o[dm][1] *= alB;
        o[dm][2] *= alA;
        o[dm][3] *= alB;
      }
    }
    const uint32_t q00 = movmatrix_trans(pack_bf16x2(p00 * beA, p01 * beB));
    const uint32_t q01 = movmatrix_trans(pack_bf16x2(p02 * beA, p03 * beB));
    const uint32_t q10 = movmatrix_trans(pack_bf16x2(p10 * beA, p11 * beB));
    const uint32_t q11 = movmatrix_trans(pack_bf16x2(p12 * beA, p13 * beB));
    const uint32_t vb0 = smem_u32(st0) + 2 * BOX_BYTES + vrow * 128;
    const uint32_t vb1 = smem_u32(st1) + 2 * BOX_BYTES + vrow * 128;
#pragma unroll
    for (int dm = 0; dm < 8; ++dm) {
      const int ch = 2 * dm + vchi;
      const uint32_t off = (ch >> 3) * BOX_BYTES + (((ch & 7) ^ xr) << 4);
      uint32_t r0, r1, r2, r3, t0, t1, t2, t3;
      ldsm_x4_trans(vb0 + off, r0, r1, r2, r3);
      ldsm_x4_trans(vb1 + off, t0, t1, t2, t3);
      mma_bf16_16816(o[dm], r0, r1, r2, r3, q00, q01);
      mma_bf16_16816(o[dm], t0, t1, t2, t3, q10, q11);
    }
  }

  // This warp's state as is, heads below r only: O^T rows into
  // so[head * ld + dim], running max and sum into sm_[head], sz_[head].
  __device__ __forceinline__ void store_state(float* so, int ld, float* sm_, float* sz_,
                                              int r) const {
    const int h0 = 2 * c4, h1 = 2 * c4 + 1;
#pragma unroll
    for (int dm = 0; dm < 8; ++dm) {
      const int d0 = dm * 16 + g4;
      if (h0 < r) {
        so[h0 * ld + d0] = o[dm][0];
        so[h0 * ld + d0 + 8] = o[dm][2];
      }
      if (h1 < r) {
        so[h1 * ld + d0] = o[dm][1];
        so[h1 * ld + d0 + 8] = o[dm][3];
      }
    }
    if (g4 == 0) {
      if (h0 < r) {
        sm_[h0] = m_run[0];
        sz_[h0] = z_run[0];
      }
      if (h1 < r) {
        sm_[h1] = m_run[1];
        sz_[h1] = z_run[1];
      }
    }
  }

  // Merge the eight warps' states pairwise into comb_*[0..NCOMB) (warps
  // cw >= NCOMB hand theirs to warp cw - NCOMB).  Called by the NT_BF16
  // consumer threads together; ends with a barrier.
  __device__ __forceinline__ void to_comb(float (*co)[GMAX][HD], float (*cm)[GMAX],
                                          float (*cz)[GMAX], int cw) {
    if (cw >= NCOMB) {
      const int w = cw - NCOMB;
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        const int d0 = dm * 16 + g4;
        co[w][2 * c4][d0] = o[dm][0];
        co[w][2 * c4 + 1][d0] = o[dm][1];
        co[w][2 * c4][d0 + 8] = o[dm][2];
        co[w][2 * c4 + 1][d0 + 8] = o[dm][3];
      }
      if (g4 == 0) {
        cm[w][2 * c4] = m_run[0];
        cm[w][2 * c4 + 1] = m_run[1];
        cz[w][2 * c4] = z_run[0];
        cz[w][2 * c4 + 1] = z_run[1];
      }
    }
    named_bar_sync(BAR_CONS, NT_BF16);
    if (cw < NCOMB) {
      const float m2A = cm[cw][2 * c4], m2B = cm[cw][2 * c4 + 1];
      const float z2A = cz[cw][2 * c4], z2B = cz[cw][2 * c4 + 1];
      __syncwarp();
      const float mnA = fmaxf(m_run[0], m2A), mnB = fmaxf(m_run[1], m2B);
      const float fA = mnA == -INFINITY ? 0.f : ex2_approx(m_run[0] - mnA);
      const float hA = mnA == -INFINITY ? 0.f : ex2_approx(m2A - mnA);
      const float fB = mnB == -INFINITY ? 0.f : ex2_approx(m_run[1] - mnB);
      const float hB = mnB == -INFINITY ? 0.f : ex2_approx(m2B - mnB);
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        const int d0 = dm * 16 + g4;
        float* a = &co[cw][2 * c4][d0];
        float* b = &co[cw][2 * c4 + 1][d0];
        a[0] = o[dm][0] * fA + a[0] * hA;
        b[0] = o[dm][1] * fB + b[0] * hB;
        a[8] = o[dm][2] * fA + a[8] * hA;
        b[8] = o[dm][3] * fB + b[8] * hB;
      }
      if (g4 == 0) {
        cm[cw][2 * c4] = mnA;
        cm[cw][2 * c4 + 1] = mnB;
        cz[cw][2 * c4] = z_run[0] * fA + z2A * hA;
        cz[cw][2 * c4 + 1] = z_run[1] * fB + z2B * hB;
      }
    }
    named_bar_sync(BAR_CONS, NT_BF16);
  }
};

// ------------------------------------------------------------ bf16 kernel

template <bool FULL>
__global__ void __launch_bounds__(NTHR_BF16, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  SmemBF16& sm = *reinterpret_cast<SmemBF16*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SmemCommon& c = sm.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&sm.fullK_bar[s], 1);
      mbar_init(&sm.fullV_bar[s], 1);
      mbar_init(&sm.empty_bar[s], NW_BF16);
      sm.bst_cnt[s] = 0;
      StageMeta z{};
      z.blk = -1;
      z.ncontrib = 1;
      sm.meta[s] = z;
    }
    c.misc[4] = 0;
    c.nseg = 0;
    c.trace_n = 0;
    c.trace_cta = (int)blockIdx.x;
    fence_mbar_init();
  }
  if (tid == 32) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  build_prefix(p, c, FULL);
  __syncthreads();
  // Work split over G = min(grid, T) CTAs so that every working CTA owns at
  // least one unit (the contributor count of a (b, h) relies on it).
  const int T = c.prefix[p.B];
  const int G = T > 0 ? min((int)gridDim.x, T) : 1;
  const int E = min(max(p.late_from, 0), G), D = late_deficit(p, T, G);
  const bool works = (int)blockIdx.x < G;
  const int lo = works ? (int)part_lo(blockIdx.x, T, G, E, D) : 0;
  const int hi = works ? (int)part_lo(blockIdx.x + 1, T, G, E, D) : 0;
  const int n = hi - lo;
  // Programmatic launch between layers.  Every global write (and a reuse
  // layer's read of indices its immediate predecessor wrote) comes after
  // griddep_wait, which returns once the preceding kernel has completed; a
  // kernel completes only after its own wait, so after a kernel's wait every
  // earlier kernel has completed.  A CTA lets the next kernel launch as soon
  // as any of its threads executes griddep_launch_dependents (the merge
  // kernel does so at once, so the next layer can start on the SMs that this
  // kernel's tail frees), and the kernel right after a reset layer (idx_wait)
  // triggers only after its wait: later reuse layers then read that reset
  // layer's indices without waiting.
  // Sequences without units get their outputs from merge_kernel.
  volatile int* abort_flag = &c.misc[4];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane != 0 || n <= 0) return;
    UnitIter it;
    it.seek(c, p, lo);
    const uint64_t pol = l2_evict_first_policy();
    const uint8_t* qbase = static_cast<const uint8_t*>(p.q);
    const uint32_t qbytes = (uint32_t)(p.r * HD * 2);
    // per-sequence values, reloaded only when the sequence changes
    int cur_b = -1, seqlen = 0;
    long long row0 = 0;
    const long long hstride = p.cap > 0 ? p.cap : p.total;
    // reused indices written by the preceding kernel: wait for it first
    bool waited = false;
    if (!FULL && p.idx_wait) {
      griddep_wait();
      waited = true;
    }
    griddep_launch_dependents();  // the producer writes nothing
    // With q_wait, the first stages' K/V tiles are requested before the wait
    // and their q rows after it (qpend: stages whose q load is deferred).
    uint32_t qpend = 0u;
    // (a deferred q load is issued even after a failed wait: its bytes are
    // counted in its stage's phase, which the drain below waits for)
    auto wait_and_flush = [&]() {
      if (waited) return;
      griddep_wait();
      waited = true;
      for (int t = 0; t < NSTAGE; ++t) {
        if (!(qpend & (1u << t))) continue;
        const StageMeta& mt = sm.meta[t];
        bulk_load(sm.qslot[t], qbase + ((size_t)mt.b * p.Hq + (size_t)mt.h * p.r) * HD * 2,
                  qbytes, &sm.fullK_bar[t]);
      }
      qpend = 0u;
    };
    int idx_cur = FULL ? 0 : unit_index_entry(p, it);
#ifdef HYLRA_TRACE
    int tn = 0;  // trace events of the producer thread
#endif
    int issued = 0;  // units 0 .. issued-1 have started their stage's phase
    for (int i = 0; i < n; ++i) {
      // after a failed wait nothing more is issued: the consumers no longer
      // wait for stages, so a refill could land in a stage still being read
      if (*abort_flag) break;
      UnitIter nx = it;
      nx.advance(c, p);
      // reuse: fetch the next unit's index now, use it next iteration
      const int idx_next = (!FULL && i + 1 < n) ? unit_index_entry(p, nx) : 0;
      if (it.b != cur_b) {
        cur_b = it.b;
        seqlen = valid_seqlen(p, cur_b, false);
        row0 = p.cap > 0 ? (long long)cur_b * p.Hkv * p.cap : p.seq_off[cur_b];
      }
      const int s = i % NSTAGE;
      const uint32_t ph = (uint32_t)((i / NSTAGE) & 1);
      // a stage is refilled only after the consumers used it, which needs q
      if (p.q_wait && i >= NSTAGE) wait_and_flush();
      if (!mbar_wait_bounded(&sm.empty_bar[s], ph ^ 1u, abort_flag, p.wait_limit)) break;
      HYLRA_TRACE_EV(tn, 256, (2 << 8) | (i & 0xff));
      const StageMeta m =
          describe_unit<FULL>(p, c, it, i, n, T, G, seqlen, FULL ? it.j : idx_cur, true);
      // the block holding the newest token is read after the wait as well
      if (p.q_wait && m.blk >= 0 && m.blk == m.nb - 1) wait_and_flush();
      sm.meta[s] = m;
      const bool seg_start = (m.flags & F_SEG_START) != 0;
      const uint32_t bytesK = (seg_start ? qbytes : 0u) + (m.blk >= 0 ? 2u * BOX_BYTES : 0u);
      const uint32_t bytesV = m.blk >= 0 ? 2u * BOX_BYTES : 0u;
      issued = i + 1;
      const int row = p.staged ? (int)(((long long)(m.b * p.Hkv + m.h) * p.k + m.pos) * BLK)
                               : (int)(row0 + (long long)m.h * hstride + (long long)m.blk * BLK);
      uint8_t* st = sm.stage[s];
      if (bytesK) {
        mbar_arrive_expect_tx(&sm.fullK_bar[s], bytesK);
        if (seg_start) {
          if (p.q_wait && !waited) {
            qpend |= 1u << s;  // loaded after the wait; into L2 now
            prefetch_l2_bulk(qbase + ((size_t)m.b * p.Hq + (size_t)m.h * p.r) * HD * 2, qbytes);
          } else
            bulk_load(sm.qslot[s], qbase + ((size_t)m.b * p.Hq + (size_t)m.h * p.r) * HD * 2,
                      qbytes, &sm.fullK_bar[s]);
        }
        if (m.blk >= 0) {
          tma_load_2d(st, &tmK, 0, row, &sm.fullK_bar[s], pol);
          tma_load_2d(st + BOX_BYTES, &tmK, 64, row, &sm.fullK_bar[s], pol);
        }
      } else {
        mbar_arrive(&sm.fullK_bar[s]);
      }
      if (bytesV) {
        mbar_arrive_expect_tx(&sm.fullV_bar[s], bytesV);
        tma_load_2d(st + 2 * BOX_BYTES, &tmV, 0, row, &sm.fullV_bar[s], pol);
        tma_load_2d(st + 3 * BOX_BYTES, &tmV, 64, row, &sm.fullV_bar[s], pol);
      } else {
        mbar_arrive(&sm.fullV_bar[s]);
      }
      it = nx;
      idx_cur = idx_next;
    }
    if (p.q_wait) wait_and_flush();
    // never exit with a copy into this CTA's shared memory in flight
    for (int t = 0; t < NSTAGE && t < issued; ++t) {
      const int last = t + (issued - 1 - t) / NSTAGE * NSTAGE;  // last unit of stage t
      const uint32_t ph = (uint32_t)((last / NSTAGE) & 1);
      if (!mbar_drain(&sm.fullK_bar[t], ph) || !mbar_drain(&sm.fullV_bar[t], ph)) *abort_flag = 1;
    }
    if (*abort_flag) atomicOr(p.status, HYLRA_STATUS_TIMEOUT);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;   // 0..7: tokens 16*cw .. 16*cw+15 of every block
  const int ct = tid - 32;
  WarpAttn wa;
  wa.init(cw, lane);
  if (FULL || !p.idx_wait) griddep_launch_dependents();  // else the producer does, after its wait
  if (p.q_wait && (FULL || !p.idx_wait) && n > 0) {
    // while q is on its way: one pass over the first staged block with a
    // zero query, result discarded (brings the code into the instruction
    // cache)
    float d0, d1, d2, d3;
    wa.block(sm.stage[0], BLK, p.scale_log2, &sm.fullV_bar[0], 0u, abort_flag, p.wait_limit, d0,
             d1, d2, d3);
    wa.reset();
  }
  bool waited = false;  // griddep_wait done (needed before the first global write)
  auto ensure_waited = [&]() {
    if (!waited) {
      griddep_wait();
      waited = true;
    }
  };
  if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, 1 << 8);
  // The consumers walk the units themselves for the segment boundaries (the
  // same walk as the producer's): every named barrier below then depends only
  // on the split, never on a stage description, so all consumer warps meet
  // the same barriers even after a failed wait left a description unwritten.
  UnitIter cit;
  if (n > 0) cit.seek(c, p, lo);

  for (int i = 0; i < n; ++i) {
    const int s = i % NSTAGE;
    const uint32_t ph = (uint32_t)((i / NSTAGE) & 1);
    const bool seg_start = i == 0 || cit.j == 0;
    const bool seg_end = i == n - 1 || cit.j == cit.U - 1;
    cit.advance(c, p);
    mbar_wait_bounded(&sm.fullK_bar[s], ph, abort_flag, p.wait_limit);
    if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, (3 << 8) | (i & 0xff));
    const StageMeta m = sm.meta[s];
    if (seg_start) {
      wa.reset();
      wa.load_q(sm.qslot[s], p.r);
    }
    if (m.blk >= 0) {
      float mxA, mxB, sA, sB;
      wa.block(sm.stage[s], m.nvalid, p.scale_log2, &sm.fullV_bar[s], ph, abort_flag,
               p.wait_limit, mxA, mxB, sA, sB);
      if (FULL && wa.g4 == 0) {
        sm.bst_s[s][cw][2 * wa.c4] = sA;
        sm.bst_s[s][cw][2 * wa.c4 + 1] = sB;
        sm.bst_m[s][cw][2 * wa.c4] = mxA;
        sm.bst_m[s][cw][2 * wa.c4 + 1] = mxB;
      }
    } else {
      mbar_wait_bounded(&sm.fullV_bar[s], ph, abort_flag, p.wait_limit);  // keep the phase in step
    }
    if (FULL && m.blk >= 0) {
      // the last warp to finish this block merges the eight shares
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(&sm.bst_cnt[s], 1) == NW_BF16 - 1;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence_block();
        ensure_waited();
        if (lane < p.r && meta_sane(p, m)) {
          float* dst = p.bstat + bstat_at(p, m.b * p.Hkv + m.h, lane, m.blk);
          float rec[2];
          combine_block_record<NW_BF16>(sm.bst_s[s], sm.bst_m[s], lane, rec);
          dst[0] = rec[0];
          dst[1] = rec[1];
        }
        if (lane == 0) sm.bst_cnt[s] = 0;
      }
    }
    __syncwarp();
    if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, (4 << 8) | (i & 0xff));
    if (lane == 0) mbar_arrive(&sm.empty_bar[s]);

    if (seg_end) {
      if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, 5 << 8);
      ensure_waited();
      wa.to_comb(c.comb_o, c.comb_m, c.comb_z, cw);  // eight warp states -> four
      store_partial<NT_BF16, false>(p, c, m, ct);  // merged by merge_kernel
      if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, 6 << 8);
    }
  }
  // every CTA waits once, so that this kernel completes only after its
  // predecessor (later kernels rely on that ordering without waiting)
  ensure_waited();
  if (ct == 0) HYLRA_TRACE_EV(c.trace_n, 0, 9 << 8);
  if (*abort_flag && ct == 0) atomicOr(p.status, HYLRA_STATUS_TIMEOUT);
}

// ------------------------------------------------------------ merge kernel
//
// Reset layers: runs after decode_bf16_kernel (as its programmatic
// dependent).  The kernel boundary makes the streaming kernel's partials
// visible; no fence or ticket is needed.  Grid (B*Hkv, 1 + merge_out_ctas(..)):
// for each (sequence, KV head) independent CTAs run side by side so that none
// waits for another and each SM loads only its share of the partials:
//   y = 0      derives each head's max and sum straight from the
//              contributors' (m, Z) pairs, scores the blocks and selects the
//              top-k;
//   y = 1..    each merges the contributors' partial rows of its heads into
//              the output.
// (Reuse layers merge in merge_reuse_kernel.)
constexpr int BAR_TOPK = 3;           // named barrier of the selection CTA

// Output CTAs per (b, h): one per head up to four when the grid stays
// within one wave of SMs (few sequences and heads: each SM then loads a
// smaller share of the partials), else one.  Heads [g0, g1) of output CTA
// `part` (1..n).
__host__ __device__ constexpr int merge_out_split(int r) {  // up to 4 CTAs, none empty
  return (r + (r + 3) / 4 - 1) / ((r + 3) / 4);
}
__host__ __device__ constexpr int merge_out_ctas(int r, long long nbh, int sms) {
  return nbh * (1 + merge_out_split(r)) <= sms ? merge_out_split(r) : 1;
}
__device__ __forceinline__ void merge_out_heads(int r, int n, int part, int& g0, int& g1) {
  const int per = (r + n - 1) / n;
  g0 = min(r, (part - 1) * per);
  g1 = min(r, g0 + per);
}

struct SmemMerge {
  float4 red[NT_MERGE];    // per-group partial rows, [group][float4 column]
  float rm[NWMAX][GMAX];   // per-group running max and sum
  float rz[NWMAX][GMAX];
  SmemCommon c;            // prefix sums; head statistics, keys and top-k scratch
};

__global__ void __launch_bounds__(NT_MERGE, 1) merge_kernel(const __grid_constant__ Params p,
                                                            int grid_stream) {
  __shared__ SmemMerge sm;
  SmemCommon& c = sm.c;
  const int tid = threadIdx.x;
  const int bh = (int)blockIdx.x;
  const int part = (int)blockIdx.y;  // 0: statistics and top-k; 1..: output heads
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int r = p.r;
  const bool outcta = part > 0;  // output rows; else statistics and top-k
  int g0 = 0, g1 = 0;
  if (outcta) {
    merge_out_heads(r, (int)gridDim.y - 1, part, g0, g1);
    if (g0 >= g1) return;  // no heads left for this part (not launched so)
  }
  // The next layer's kernel may launch now: it reads nothing of this layer
  // and writes nothing before its own wait, which returns only after this
  // kernel, and so the streaming kernel, has completed.  Its CTAs take the
  // SMs the streaming kernel's tail frees and start staging their tiles.
  griddep_launch_dependents();
  if (tid == 0) {
    c.trace_n = 0;
    c.trace_cta = 160 + bh * 8 + part;
    HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 30 << 8);
  }
  // everything that does not depend on the streaming kernel's output first
  build_prefix(p, c, true);
  const int seqlen = valid_seqlen(p, b, false);
  __syncthreads();
  const int T = c.prefix[p.B];
  const int U = (c.prefix[b + 1] - c.prefix[b]) / p.Hkv;
  const int G = min(grid_stream, max(T, 1));
  const int E = min(max(p.late_from, 0), G), D = late_deficit(p, T, G);
  const int start = c.prefix[b] + h * U;
  int first = 0, nc = 0;
  if (U > 0) {
    // the streaming kernel's static split (part_lo): every CTA of it owns
    // at least one unit, so the owners of (b, h) are contiguous
    first = part_owner(start, T, G, E, D);
    nc = part_owner((long long)start + U - 1, T, G, E, D) - first + 1;
    first += bh;  // partial slot of contributor c is c + bh
  }
  const int nb = (seqlen + BLK - 1) / BLK;
  const float* pbase = p.partials + (size_t)first * SLOT_FLOATS;
  float* out_bh = p.out + ((size_t)b * p.Hq + (size_t)h * r) * HD;
  if (U > 0 && tid < 6) {
    // Before the wait: a line at each end of every range read or written
    // after it, so that their address translations are cached when it
    // returns (values discarded: nothing is used before the wait).
    const int32_t* idx_row = p.topk_out + (size_t)bh * p.k;
    const void* ptr;
    if (!outcta) {
      const float* bs0 = p.bstat + bstat_at(p, bh, 0, 0);
      const float* bs1 = p.bstat + bstat_at(p, bh, r - 1, max(nb - 1, 0)) + 1;
      ptr = tid == 0 ? (const void*)bs0
          : tid == 1 ? (const void*)bs1
          : tid == 2 ? (const void*)idx_row
          : tid == 3 ? (const void*)(idx_row + max(p.k - 1, 0))
          : tid == 4 ? (const void*)(pbase + GMAX * HD)
                     : (const void*)(pbase + (size_t)nc * SLOT_FLOATS - 1);
    } else {
      ptr = tid == 0 ? (const void*)pbase
          : tid == 1 ? (const void*)(pbase + (size_t)nc * SLOT_FLOATS - 1)
          : tid == 2 ? (const void*)(out_bh + g0 * HD)
          : tid == 3 ? (const void*)(out_bh + g1 * HD - 1)
          : tid == 4 ? (const void*)(pbase + (size_t)(nc / 2) * SLOT_FLOATS)
                     : (const void*)(pbase + (size_t)(nc - 1) * SLOT_FLOATS);
    }
    touch_line(ptr);
  }
  griddep_wait();  // the streaming kernel has completed: partials are visible
  if (tid == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 31 << 8);
  if (U == 0) {
    // a sequence without units: zero output (and no indices)
    if (outcta)
      for (int i = g0 * HD + tid; i < g1 * HD; i += NT_MERGE) out_bh[i] = 0.f;
    else
      for (int i = tid; i < p.k; i += NT_MERGE) p.topk_out[(size_t)bh * p.k + i] = -1;
    return;
  }

  if (outcta) {
    // ------------------------------------------ output rows g0..g1-1 (LSE merge)
    constexpr int CB = 10;  // contributors per thread and batch of loads
    const int ncol = (g1 - g0) * (HD / 4);  // float4 columns
    const int GA = ncol >= NT_MERGE ? 1 : min(NWMAX, NT_MERGE / ncol);
    for (int t = tid; t < GA * ncol; t += NT_MERGE) {
      const int q = t / ncol, col = t - q * ncol;
      const int g = g0 + col / (HD / 4), d4 = col % (HD / 4);
      float M = -INFINITY, Z = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = q; j0 < nc; j0 += GA * CB) {
        float mv[CB], zv[CB];
        float4 ov[CB];
#pragma unroll
        for (int u = 0; u < CB; ++u) {
          const int j = j0 + u * GA;  // the same in every lane of a warp
          mv[u] = -INFINITY;
          if (j < nc) {
            const float* sl = pbase + (size_t)j * SLOT_FLOATS;
            mv[u] = __ldcg(sl + GMAX * HD + g);
            zv[u] = __ldcg(sl + GMAX * HD + GMAX + g);
            ov[u] = __ldcg(reinterpret_cast<const float4*>(sl + g * HD + 4 * d4));
          }
        }
        float mb = M;
#pragma unroll
        for (int u = 0; u < CB; ++u) mb = fmaxf(mb, mv[u]);
        if (mb != -INFINITY) {
          const float fo = M == -INFINITY ? 0.f : ex2_approx(M - mb);
          acc.x *= fo;
          acc.y *= fo;
          acc.z *= fo;
          acc.w *= fo;
          Z *= fo;
#pragma unroll
          for (int u = 0; u < CB; ++u) {
            if (mv[u] == -INFINITY) continue;
            const float f = ex2_approx(mv[u] - mb);
            acc.x = fmaf(ov[u].x, f, acc.x);
            acc.y = fmaf(ov[u].y, f, acc.y);
            acc.z = fmaf(ov[u].z, f, acc.z);
            acc.w = fmaf(ov[u].w, f, acc.w);
            Z = fmaf(zv[u], f, Z);
          }
          M = mb;
        }
      }
      sm.red[t] = acc;
      if (d4 == 0) {
        sm.rm[q][g] = M;
        sm.rz[q][g] = Z;
      }
    }
    __syncthreads();
    if (tid == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 24 << 8);
    for (int col = tid; col < ncol; col += NT_MERGE) {
      const int g = g0 + col / (HD / 4), d4 = col % (HD / 4);
      float M = -INFINITY;
      for (int q = 0; q < GA; ++q) M = fmaxf(M, sm.rm[q][g]);
      float Z = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
        for (int q = 0; q < GA; ++q) {
          const float mq = sm.rm[q][g];
          if (mq == -INFINITY) continue;
          const float f = ex2_approx(mq - M);
          const float4 v = sm.red[q * ncol + col];
          acc.x = fmaf(v.x, f, acc.x);
          acc.y = fmaf(v.y, f, acc.y);
          acc.z = fmaf(v.z, f, acc.z);
          acc.w = fmaf(v.w, f, acc.w);
          Z = fmaf(sm.rz[q][g], f, Z);
        }
      }
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (Z > 0.f) o = make_float4(acc.x / Z, acc.y / Z, acc.z / Z, acc.w / Z);
      *reinterpret_cast<float4*>(out_bh + g * HD + 4 * d4) = o;
    }
    if (tid == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 17 << 8);
    return;
  }

  const int tb = tid;  // 0..NT_MERGE-1
  const int wb = tb >> 5, lane = tb & 31;
  {
    // --------------------------------------------- block scores and top-k
    // block records of this thread's first SPT blocks (tb, tb + 256, ...),
    // all loaded up front, together with the head statistics below
    // (the conditions are the same in every lane of a warp and lanes past
    // the last block reload it, so no load result selects against a
    // default, which would wait for that load on the spot; entries g >= r
    // and blocks past nb are never read)
    constexpr int SPT = 4;
    float2 sv0[SPT][GMAX];
#pragma unroll
    for (int u = 0; u < SPT; ++u) {
      if (u * NT_MERGE + wb * 32 < nb) {
        const int beta = min(tb + u * NT_MERGE, nb - 1);
#pragma unroll
        for (int g = 0; g < GMAX; ++g)
          if (g < r)
            sv0[u][g] =
                __ldcg(reinterpret_cast<const float2*>(p.bstat + bstat_at(p, bh, g, beta)));
      }
    }
    // head g's max and sum, straight from the contributors' (m, Z): warp g
    // (a (b, h) has at most MAX_CTAS contributors)
    if (wb < r) {
      const int g = wb;
      float mj[MAX_CTAS / 32], zj[MAX_CTAS / 32];
      float M = -INFINITY;
#pragma unroll
      for (int u = 0; u < MAX_CTAS / 32; ++u) {
        if (u * 32 < nc) {  // warp-uniform; lanes past nc reload the last one
          const float* sl = pbase + (size_t)min(u * 32 + lane, nc - 1) * SLOT_FLOATS;
          mj[u] = __ldcg(sl + GMAX * HD + g);
          zj[u] = __ldcg(sl + GMAX * HD + GMAX + g);
        }
      }
#pragma unroll
      for (int u = 0; u < MAX_CTAS / 32; ++u) {
        if (u * 32 + lane >= nc) {
          mj[u] = -INFINITY;
          zj[u] = 0.f;
        }
        M = fmaxf(M, mj[u]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      if (tb == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 19 << 8);
      float Z = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int u = 0; u < MAX_CTAS / 32; ++u)
          if (mj[u] != -INFINITY) Z = fmaf(zj[u], ex2_approx(mj[u] - M), Z);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, off);
      if (lane == 0) {
        c.mg[g] = M;
        c.zg[g] = Z;
        c.rzg[g] = Z > 0.f ? 1.f / Z : 0.f;
      }
    }
    named_bar_sync(BAR_TOPK, NT_MERGE);
    if (tb == 0) HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 18 << 8);
    // score of block beta: its attention mass summed over the r heads
    uint32_t* keys = reinterpret_cast<uint32_t*>(&c.comb_o[0][0][0]);
    bool nonfinite = false;
    auto score_key = [&](const float2 (&sv)[GMAX]) {
      float score = 0.f;
#pragma unroll
      for (int g = 0; g < GMAX; ++g)
        if (g < r && c.zg[g] > 0.f && sv[g].y != -INFINITY)
          score += sv[g].x * exp2f(sv[g].y - c.mg[g]) * c.rzg[g];
      uint32_t key = 0u;
      if (isfinite(score)) {
        if (score > 0.f) key = __float_as_uint(score);
      } else {
        nonfinite = true;
      }
      return key;
    };
#pragma unroll
    for (int u = 0; u < SPT; ++u) {
      const int beta = tb + u * NT_MERGE;
      if (beta < nb) keys[beta] = score_key(sv0[u]);
    }
    for (int beta = tb + SPT * NT_MERGE; beta < nb; beta += NT_MERGE) {
      float2 sv[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g)
        sv[g] = g < r ? __ldcg(reinterpret_cast<const float2*>(
                            p.bstat + bstat_at(p, bh, g, beta)))
                      : make_float2(0.f, -INFINITY);
      keys[beta] = score_key(sv);
    }
    if (nonfinite) atomicOr(p.status, HYLRA_STATUS_NONFINITE);
    named_bar_sync(BAR_TOPK, NT_MERGE);
    if (tb == 0) {
      HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 12 << 8);
      HYLRA_TRACE_VAL(c.trace_n, c.trace_cta, 43 << 8, HYLRA_CLOCK());
    }
    topk_select<NT_MERGE, BAR_TOPK>(p, c, bh, nb, tb);
    if (tb == 0) {
      HYLRA_TRACE_VAL(c.trace_n, c.trace_cta, 44 << 8, HYLRA_CLOCK());
      HYLRA_TRACE_CTA(c.trace_n, c.trace_cta, 13 << 8);
    }
  }
}

// ------------------------------------------------------ reuse merge kernel
//
// Reuse layers on the bf16 streaming kernel: its programmatic dependent, one
// CTA of NT_RMERGE threads per (b, h) that LSE-merges the contributors'
// partial rows into the output and checks the index list for repeats.  Its
// CTAs start on SMs that this layer's streaming CTAs leave and wait there for
// the layer to end; an SM that holds one cannot take a streaming CTA of the
// next layer (the nine warps of a streaming CTA leave too few registers in
// one SM sub-partition for any other CTA beside them, and too little shared
// memory beside a larger one).  So the CTA is small (four warps, under 100
// registers a thread, 272 bytes of shared memory: five share an SM) and
// holds as few of the SMs that the next layer's CTAs wait for as it can.
constexpr int NT_RMERGE = 128;

__global__ void __launch_bounds__(NT_RMERGE, 4) merge_reuse_kernel(const __grid_constant__ Params p,
                                                                  int grid_stream) {
  __shared__ uint32_t seen[MAX_NB / 32];  // blocks named so far in the index list
  __shared__ int units[2];                // units before sequence b (all heads), all units
  const int tid = threadIdx.x, lane = tid & 31;
  const int bh = (int)blockIdx.x;
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int r = p.r;
  // the next layer's kernel may launch now (as in merge_kernel)
  griddep_launch_dependents();
#ifdef HYLRA_TRACE
  int tn = 0;
  const int tcta = 160 + bh;
  if (tid == 0) HYLRA_TRACE_CTA(tn, tcta, 30 << 8);
#endif
  // everything that does not depend on the streaming kernel's output first:
  // the unit counts (warp 0, no per-sequence array) and the split
  if (tid < 32) {
    int before = 0, total = 0;
    for (int s = lane; s < p.B; s += 32) {
      const int n = units_of(p, valid_seqlen(p, s, false), false) * p.Hkv;
      total += n;
      if (s < b) before += n;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, off);
      total += __shfl_xor_sync(0xffffffffu, total, off);
    }
    if (lane == 0) {
      units[0] = before;
      units[1] = total;
    }
  }
  for (int i = tid; i < MAX_NB / 32; i += NT_RMERGE) seen[i] = 0u;
  const int seqlen = valid_seqlen(p, b, false);
  __syncthreads();
  const int T = units[1];
  const int nb = (seqlen + BLK - 1) / BLK;
  const int U = units_of(p, seqlen, false);
  const int kp = min(p.k, nb);
  const int G = min(grid_stream, max(T, 1));
  const int E = min(max(p.late_from, 0), G), D = late_deficit(p, T, G);
  const int start = units[0] + h * U;
  int first = 0, nc = 0;
  if (U > 0) {
    // the streaming kernel's static split (part_lo): every CTA of it owns
    // at least one unit, so the owners of (b, h) are contiguous
    first = part_owner(start, T, G, E, D);
    nc = part_owner((long long)start + U - 1, T, G, E, D) - first + 1;
    first += bh;  // partial slot of contributor c is c + bh
  }
  const float* pbase = p.partials + (size_t)first * SLOT_FLOATS;
  float* out_bh = p.out + ((size_t)b * p.Hq + (size_t)h * r) * HD;
  const int32_t* idx = p.topk_in + (size_t)bh * p.k;
  if (U > 0 && tid < 4) {
    // before the wait: a line at each end of the ranges read or written after
    // it (address translations; values discarded)
    const void* ptr = tid == 0 ? (const void*)pbase
                    : tid == 1 ? (const void*)(pbase + (size_t)nc * SLOT_FLOATS - 1)
                    : tid == 2 ? (const void*)out_bh
                               : (const void*)(out_bh + r * HD - 1);
    touch_line(ptr);
  }
  griddep_wait();  // the streaming kernel has completed: partials are visible
#ifdef HYLRA_TRACE
  if (tid == 0) HYLRA_TRACE_CTA(tn, tcta, 31 << 8);
#endif
  if (U == 0) {
    // a sequence without units: zero output
    for (int i = tid; i < r * HD; i += NT_RMERGE) out_bh[i] = 0.f;
    return;
  }
  // this thread's entries of the index list, loaded together with the partials
  constexpr int EPT = HYLRA_MAX_TOPK / NT_RMERGE;
  int32_t ent[EPT];
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int e = tid + u * NT_RMERGE;
    ent[u] = e < kp ? __ldcg(idx + e) : -1;
  }
  // output rows: thread t merges float4 column t (and t + 128 when r > 4)
  // over every contributor, online, in batches of CB loads
  constexpr int CB = 8;
  for (int col = tid; col < r * (HD / 4); col += NT_RMERGE) {
    const int g = col / (HD / 4), d4 = col % (HD / 4);
    float M = -INFINITY, Z = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < nc; j0 += CB) {
      float mv[CB], zv[CB];
      float4 ov[CB];
#pragma unroll
      for (int u = 0; u < CB; ++u) {
        const int j = j0 + u;  // the same in every thread
        mv[u] = -INFINITY;
        if (j < nc) {
          const float* sl = pbase + (size_t)j * SLOT_FLOATS;
          mv[u] = __ldcg(sl + GMAX * HD + g);
          zv[u] = __ldcg(sl + GMAX * HD + GMAX + g);
          ov[u] = __ldcg(reinterpret_cast<const float4*>(sl + g * HD + 4 * d4));
        }
      }
      float mb = M;
#pragma unroll
      for (int u = 0; u < CB; ++u) mb = fmaxf(mb, mv[u]);
      if (mb != -INFINITY) {
        const float fo = M == -INFINITY ? 0.f : ex2_approx(M - mb);
        acc.x *= fo;
        acc.y *= fo;
        acc.z *= fo;
        acc.w *= fo;
        Z *= fo;
#pragma unroll
        for (int u = 0; u < CB; ++u) {
          if (mv[u] == -INFINITY) continue;
          const float f = ex2_approx(mv[u] - mb);
          acc.x = fmaf(ov[u].x, f, acc.x);
          acc.y = fmaf(ov[u].y, f, acc.y);
          acc.z = fmaf(ov[u].z, f, acc.z);
          acc.w = fmaf(ov[u].w, f, acc.w);
          Z = fmaf(zv[u], f, Z);
        }
        M = mb;
      }
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (Z > 0.f) o = make_float4(acc.x / Z, acc.y / Z, acc.z / Z, acc.w / Z);
    *reinterpret_cast<float4*>(out_bh + g * HD + 4 * d4) = o;
  }
  // a reused list naming one block twice counts that block twice: flag it
  // (entries outside the sequence are skipped and flagged by the streaming
  // kernel)
  bool dup = false;
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int32_t v = ent[u];
    if (v >= 0 && v < nb) {
      const uint32_t bit = 1u << (v & 31);
      dup |= (atomicOr(&seen[v >> 5], bit) & bit) != 0u;
    }
  }
  if (dup) atomicOr(p.status, HYLRA_STATUS_DUP_INDEX);
#ifdef HYLRA_TRACE
  if (tid == 0) HYLRA_TRACE_CTA(tn, tcta, 17 << 8);
#endif
}

// ------------------------------------------------- cluster reuse kernel
//
// Reuse layers touch only k' blocks per (sequence, KV head), too little data
// to hide a cross-CTA merge through global memory.  Here the CTAs sharing a
// (b, h) form one thread-block cluster (grid = cluster size x B*Hkv): CTA
// `rank` takes blocks rank*upc .. rank*upc+upc-1 of the index list, merges
// its warps' states, and stores the result straight into slot `rank` of
// CTA 0's shared memory (distributed shared memory stores are posted, so
// they pipeline; loads from a peer CTA do not).  One cluster barrier later
// CTA 0 merges the slots from its own shared memory and writes the output.
// No workspace, fence or ticket is involved, and every CTA but rank 0
// leaves right after its stores.

constexpr int NST_MAX_RC = 3;

struct SmemRC {
  uint8_t qbuf[QSLOT_BYTES];
  int meta_blk[NST_MAX_RC];
  int meta_nvalid[NST_MAX_RC];
  alignas(8) uint64_t fullK_bar[NST_MAX_RC];
  alignas(8) uint64_t fullV_bar[NST_MAX_RC];
  alignas(8) uint64_t empty_bar[NST_MAX_RC];
  alignas(8) uint64_t gather_bar;  // rank 0: every CTA's slot has arrived
  uint32_t seen[MAX_NB / 32];      // rank 0: blocks named so far (duplicate check)
  int abort_flag;
};

// The eight consumer warps' states: O^T rows [warp][head < r][RC_LD] (the
// row pitch of HD + 4 floats spreads a warp's stores over all banks), then
// running max and sum [warp][GMAX] each.
constexpr int RC_LD = HD + 4;

// Per-CTA slot in rank 0's gather area: O[r][HD] (unnormalised), then
// (m, Z) per head; only the first 4 r (HD + 2) bytes are sent.
__host__ __device__ constexpr int rc_slot_floats(int r) { return r * HD + 2 * GMAX; }
__host__ __device__ constexpr uint32_t rc_slot_bytes_sent(int r) { return 4u * r * (HD + 2); }

// Dynamic shared memory: header | gather (cs slots) | warp states | nst
// stages, each part 1024-byte aligned (the stages hold 128-byte-swizzled
// TMA tiles).
__host__ __device__ constexpr size_t rc_align(size_t x) { return (x + 1023) / 1024 * 1024; }
__host__ __device__ constexpr size_t rc_header_bytes() { return rc_align(sizeof(SmemRC)); }
__host__ __device__ constexpr size_t rc_gather_bytes(int cs, int r) {
  return rc_align((size_t)cs * rc_slot_floats(r) * 4);
}
__host__ __device__ constexpr size_t rc_comb_bytes(int r) {
  return rc_align((size_t)NW_BF16 * (r * RC_LD + 2 * GMAX) * 4);
}
// With comb_in_stage the warp states go to stage 0, which every consumer
// warp is done with by then (a barrier first); that leaves room for one more
// stage when blocks outnumber stages.
__host__ __device__ constexpr size_t rc_smem_bytes(int cs, int r, int nst,
                                                   bool comb_in_stage = false) {
  return rc_header_bytes() + rc_gather_bytes(cs, r) + (comb_in_stage ? 0 : rc_comb_bytes(r)) +
         (size_t)nst * STAGE_BYTES;
}

// One output pair (head g, columns col, col+1) from the first cs of NS
// gather slots: every slot's (m, Z) and O pair loaded at once.
template <int NS>
__device__ __forceinline__ float2 rc_merge_pair(const float* gather, int slot, int cs, int r,
                                                int g, int col) {
  float2 mz[NS], v[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    mz[j] = make_float2(-INFINITY, 0.f);
    v[j] = make_float2(0.f, 0.f);
    if (j < cs) {
      const float* sl = gather + j * slot;
      mz[j] = *reinterpret_cast<const float2*>(sl + r * HD + 2 * g);
      v[j] = *reinterpret_cast<const float2*>(sl + g * HD + col);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int j = 0; j < NS; ++j) M = fmaxf(M, mz[j].x);
  float Z = 0.f, a0 = 0.f, a1 = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      const float f = mz[j].x == -INFINITY ? 0.f : ex2_approx(mz[j].x - M);
      Z = fmaf(mz[j].y, f, Z);
      a0 = fmaf(v[j].x, f, a0);
      a1 = fmaf(v[j].y, f, a1);
    }
  }
  return Z > 0.f ? make_float2(a0 / Z, a1 / Z) : make_float2(0.f, 0.f);
}

__global__ void __launch_bounds__(NTHR_BF16, 1)
    decode_reuse_cluster_kernel(const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV,
                                const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SmemRC& sm = *reinterpret_cast<SmemRC*>(base);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CS = (int)gridDim.x;
  const int r = p.r;
  float* gather = reinterpret_cast<float*>(base + rc_header_bytes());
  uint8_t* after_gather = base + rc_header_bytes() + rc_gather_bytes(CS, r);
  uint8_t* stages = after_gather + (p.comb_in_stage ? 0 : rc_comb_bytes(r));
  float* comb_o = reinterpret_cast<float*>(p.comb_in_stage ? stages : after_gather);
  float* comb_m = comb_o + NW_BF16 * r * RC_LD;  // [warp][GMAX]
  float* comb_z = comb_m + NW_BF16 * GMAX;
  const uint32_t rank = cluster_ctarank();
  const int bh = (int)blockIdx.y;
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int nst = p.nst, upc = p.upc;
  const int slot = rc_slot_floats(r);

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&sm.fullK_bar[s], 1);
      mbar_init(&sm.fullV_bar[s], 1);
      mbar_init(&sm.empty_bar[s], NW_BF16);
      // a consumer that gave up waiting reads a description that the
      // producer may not have written: start from "no block"
      sm.meta_blk[s] = -1;
      sm.meta_nvalid[s] = 0;
    }
    if (rank == 0) {
      // completes once every CTA's slot has landed (st.async transactions)
      mbar_init(&sm.gather_bar, 1);
      mbar_arrive_expect_tx(&sm.gather_bar, (uint32_t)CS * rc_slot_bytes_sent(r));
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid == 32) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  __syncthreads();
  // first phase of the cluster barrier: every CTA has started (waited on
  // before the first store into a peer's shared memory)
  cluster_arrive_relaxed();
  volatile int* abort_flag = &sm.abort_flag;
  const int seqlen = valid_seqlen(p, b, rank == 0 && h == 0 && tid == 0);
  const int nb = (seqlen + BLK - 1) / BLK;
  const int kp = min(p.k, nb);
  const int j0 = (int)rank * upc;
  const int nu = max(0, min(upc, kp - j0));  // blocks of this CTA
  const int tcta = bh * CS + (int)rank;
#ifdef HYLRA_TRACE
  int tn = 0;  // trace events of the first consumer thread
#endif
  (void)tcta;
  if (tid == 32) {
    HYLRA_TRACE_CTA(tn, tcta, 1 << 8);
    HYLRA_TRACE_VAL(tn, tcta, 41 << 8, HYLRA_CLOCK());
  }
  const uint8_t* qsrc =
      static_cast<const uint8_t*>(p.q) + ((size_t)b * p.Hq + (size_t)h * r) * HD * 2;
  const uint32_t qbytes = (uint32_t)(r * HD * 2);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // With q_wait the query (and the block holding the newest token) come
    // from the preceding kernel: they are read after griddep_wait.  Before
    // it, the K/V tiles of the first nst blocks are requested, and q and
    // everything else this CTA will read are brought into L2.
    const int32_t* idx = p.topk_in + (size_t)bh * p.k;
    bool waited = false;
    if (p.idx_wait) {
      // warm the index row's address translation before the wait
      if (lane == 0) touch_line(idx + j0);
      griddep_wait();  // indices written by the preceding kernel
      waited = true;
    }
    if (lane == 0 && p.q_wait && !waited) prefetch_l2_bulk(qsrc, qbytes);
    // this CTA's first 32 indices, one per lane, in one round trip
    int my_blk = lane < nu ? __ldcg(idx + j0 + lane) : -1;
    if (rank == 0) {
      // a reused list naming one block twice counts that block twice: flag it
      for (int i = lane; i < MAX_NB / 32; i += 32) sm.seen[i] = 0u;
      __syncwarp();
      bool dup = false;
      for (int e = lane; e < kp; e += 32) {
        const int32_t v = e < nu && e < 32 ? my_blk : __ldcg(idx + e);  // rank 0: j0 = 0
        if (v >= 0 && v < nb) {
          const uint32_t bit = 1u << (v & 31);
          dup |= (atomicOr(&sm.seen[v >> 5], bit) & bit) != 0u;
        }
      }
      if (__any_sync(0xffffffffu, dup) && lane == 0) atomicOr(p.status, HYLRA_STATUS_DUP_INDEX);
    }
    griddep_launch_dependents();  // the producer writes nothing
#ifdef HYLRA_TRACE
    int tp = 128;  // trace events of the producer thread
#endif
    if (lane == 0) HYLRA_TRACE_CTA(tp, tcta, 2 << 8);
    const uint64_t pol = l2_evict_first_policy();
    const long long row0 = row_base(p, b, h);
    // blocks beyond the pipeline depth (and, with q_wait, the newest block)
    // into L2 now: lane i holds this CTA's i-th block
    auto unit_row = [&](int i, int blk) -> int {
      return p.staged ? (int)(((long long)bh * p.k + j0 + i) * BLK) : (int)(row0 + (long long)blk * BLK);
    };
    if (lane < nu && my_blk >= 0 && my_blk < nb && lane >= nst) {
      const int row = unit_row(lane, my_blk);
      tma_prefetch_l2_2d(&tmK, 0, row);
      tma_prefetch_l2_2d(&tmK, 64, row);
      tma_prefetch_l2_2d(&tmV, 0, row);
      tma_prefetch_l2_2d(&tmV, 64, row);
    }
    int qpend = 0;
    int issued = 0;  // blocks 0 .. issued-1 have started their stage's phase
    for (int i = 0; i < nu; ++i) {
      const int s = i % nst;
      const uint32_t ph = (uint32_t)((i / nst) & 1);
      // after a failed wait nothing more is issued (the whole warp stops)
      if (__shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0)) break;
      int blk = i < 32 ? __shfl_sync(0xffffffffu, my_blk, i) : 0;
      if (lane != 0) continue;
      if (i >= 32) blk = __ldcg(idx + j0 + i);
      if (blk < 0 || blk >= nb) {
        if (blk != -1) atomicOr(p.status, HYLRA_STATUS_BAD_INDEX);
        blk = -1;
      }
      // a stage is refilled only after the consumers used it, which needs q
      // (the block holding the newest token is staged early like the rest:
      // its consumer warp rewrites the newest row after the wait)
      // (a deferred q load is issued even after a failed wait: its bytes are
      // counted in stage 0's first phase, which the drain below waits for)
      if (p.q_wait && !waited && i >= nst) {
        griddep_wait();
        waited = true;
        if (qpend) bulk_load(sm.qbuf, qsrc, qbytes, &sm.fullK_bar[0]);
        qpend = 0;
      }
      if (!mbar_wait_bounded(&sm.empty_bar[s], ph ^ 1u, abort_flag, p.wait_limit)) continue;
      sm.meta_blk[s] = blk;
      sm.meta_nvalid[s] = blk >= 0 ? min(BLK, seqlen - blk * BLK) : 0;
      const uint32_t bytesK = (i == 0 ? qbytes : 0u) + (blk >= 0 ? 2u * BOX_BYTES : 0u);
      const uint32_t bytesV = blk >= 0 ? 2u * BOX_BYTES : 0u;
      issued = i + 1;
      uint8_t* st = stages + (size_t)s * STAGE_BYTES;
      const int row = unit_row(i, blk);
      if (bytesK) {
        mbar_arrive_expect_tx(&sm.fullK_bar[s], bytesK);
        if (i == 0) {
          if (p.q_wait && !waited)
            qpend = 1;
          else
            bulk_load(sm.qbuf, qsrc, qbytes, &sm.fullK_bar[s]);
        }
        if (blk >= 0) {
          tma_load_2d(st, &tmK, 0, row, &sm.fullK_bar[s], pol);
          tma_load_2d(st + BOX_BYTES, &tmK, 64, row, &sm.fullK_bar[s], pol);
        }
      } else {
        mbar_arrive(&sm.fullK_bar[s]);
      }
      if (bytesV) {
        mbar_arrive_expect_tx(&sm.fullV_bar[s], bytesV);
        tma_load_2d(st + 2 * BOX_BYTES, &tmV, 0, row, &sm.fullV_bar[s], pol);
        tma_load_2d(st + 3 * BOX_BYTES, &tmV, 64, row, &sm.fullV_bar[s], pol);
      } else {
        mbar_arrive(&sm.fullV_bar[s]);
      }
      HYLRA_TRACE_CTA(tp, tcta, (12 << 8) | (i & 0x7f) | (waited ? 0x80 : 0));
    }
    if (lane == 0 && p.q_wait && !waited) {
      griddep_wait();
      if (qpend) bulk_load(sm.qbuf, qsrc, qbytes, &sm.fullK_bar[0]);
    }
    // never exit with a copy into this CTA's shared memory in flight
    if (lane == 0) {
      for (int t = 0; t < nst && t < issued; ++t) {
        const int last = t + (issued - 1 - t) / nst * nst;  // last block of stage t
        const uint32_t ph = (uint32_t)((last / nst) & 1);
        if (!mbar_drain(&sm.fullK_bar[t], ph) || !mbar_drain(&sm.fullV_bar[t], ph))
          *abort_flag = 1;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1;
    const int ct = tid - 32;
    // consumers write nothing before rank 0's griddep_wait; with idx_wait the
    // producer triggers, after its own wait
    if (!p.idx_wait) griddep_launch_dependents();
    WarpAttn wa;
    wa.init(cw, lane);
    // With q_wait the newest row of the sequence (written by the preceding
    // kernel in a model) is re-read after the wait by the one warp whose 16
    // rows hold it (each warp reads only its own rows of a stage): one
    // 16-byte chunk of K or V per lane, into its swizzled place.
    const long long row0c = (p.q_wait && !p.staged) ? row_base(p, b, h) : 0;
    auto patch_newest = [&](int s, uint32_t ph) {
      const int blk = sm.meta_blk[s];
      if (!p.q_wait || p.staged || blk < 0 || blk != nb - 1) return;
      // the newest row within the block, from the length itself (not from the
      // stage description, which a failed wait may leave half written)
      const int rr = seqlen - 1 - blk * BLK;
      if ((rr >> 4) != cw) return;
      mbar_wait_bounded(&sm.fullV_bar[s], ph, abort_flag, p.wait_limit);  // V landed (K: fullK)
      griddep_wait();
      const int c = lane & 15;
      const long long grow = row0c + (long long)blk * BLK + rr;
      const uint8_t* src =
          static_cast<const uint8_t*>(lane < 16 ? p.K : p.V) + grow * (HD * 2) + c * 16;
      uint8_t* dst = stages + (size_t)s * STAGE_BYTES + (lane < 16 ? 0 : 2 * BOX_BYTES) +
                     (c >> 3) * BOX_BYTES + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
      if (!*abort_flag) *reinterpret_cast<uint4*>(dst) = __ldcg(reinterpret_cast<const uint4*>(src));
      // the stage may be released and refilled by TMA (async proxy) later:
      // order this generic-proxy write before any such refill
      fence_proxy_async_smem();
      __syncwarp();
    };
    // first phase of the cluster barrier (every CTA has started), needed
    // before the stores into CTA 0; taken now, while the data is on its way
    cluster_wait_acquire();
    if (rank == 0 && ct == 0)  // the output row's address translation
      touch_line(p.out + ((size_t)b * p.Hq + (size_t)h * r) * HD);
    // Blocks go in pairs (one 256-token step each) when every block has its
    // own stage; with refills, one at a time so each freed stage reloads
    // early.  A stage is released only when a refill follows.
    int i = 0;
    for (; nu <= nst && i + 1 < nu; i += 2) {
      const int s0 = i % nst, s1 = (i + 1) % nst;
      const uint32_t ph0 = (uint32_t)((i / nst) & 1), ph1 = (uint32_t)(((i + 1) / nst) & 1);
      mbar_wait_bounded(&sm.fullK_bar[s0], ph0, abort_flag, p.wait_limit);
      mbar_wait_bounded(&sm.fullK_bar[s1], ph1, abort_flag, p.wait_limit);
      if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 3 << 8);
      if (i == 0) wa.load_q(sm.qbuf, r);
      const int blk0 = sm.meta_blk[s0], blk1 = sm.meta_blk[s1];
      const int nv0 = sm.meta_nvalid[s0], nv1 = sm.meta_nvalid[s1];
      if (blk0 == nb - 1) patch_newest(s0, ph0);
      if (blk1 == nb - 1) patch_newest(s1, ph1);
      wa.block2(stages + (size_t)s0 * STAGE_BYTES, nv0, &sm.fullV_bar[s0], ph0,
                stages + (size_t)s1 * STAGE_BYTES, nv1, &sm.fullV_bar[s1], ph1, p.scale_log2,
                abort_flag, p.wait_limit);
    }
    for (; i < nu; ++i) {
      const int s = i % nst;
      const uint32_t ph = (uint32_t)((i / nst) & 1);
      mbar_wait_bounded(&sm.fullK_bar[s], ph, abort_flag, p.wait_limit);
      if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 3 << 8);
      if (i == 0) wa.load_q(sm.qbuf, r);
      const int blk = sm.meta_blk[s];
      if (blk == nb - 1) patch_newest(s, ph);
      if (blk >= 0) {
        float mxA, mxB, sA, sB;
        wa.block(stages + (size_t)s * STAGE_BYTES, sm.meta_nvalid[s], p.scale_log2,
                 &sm.fullV_bar[s], ph, abort_flag, p.wait_limit, mxA, mxB, sA, sB);
      } else {
        mbar_wait_bounded(&sm.fullV_bar[s], ph, abort_flag, p.wait_limit);
      }
      if (i + nst < nu) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty_bar[s]);
      }
    }
    if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 4 << 8);
    // this CTA's state: the eight warp states merged into one and sent to
    // slot `rank` of CTA 0's gather area (st.async: the bytes complete CTA
    // 0's gather barrier, so no cluster barrier is needed afterwards)
    if (p.comb_in_stage) named_bar_sync(BAR_CONS, NT_BF16);  // stage 0 no longer read
    wa.store_state(comb_o + cw * r * RC_LD, RC_LD, comb_m + cw * GMAX, comb_z + cw * GMAX, r);
    named_bar_sync(BAR_CONS, NT_BF16);
    const uint32_t dst = mapa_shared(smem_u32(gather), 0u) + (uint32_t)((int)rank * slot) * 4u;
    const uint32_t gbar = mapa_shared(smem_u32(&sm.gather_bar), 0u);
    for (int pr = ct; pr < r * (HD / 2); pr += NT_BF16) {
      const int g = pr / (HD / 2), col = 2 * (pr % (HD / 2));
      float mw[NW_BF16];
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW_BF16; ++w) {
        mw[w] = comb_m[w * GMAX + g];
        M = fmaxf(M, mw[w]);
      }
      float o0 = 0.f, o1 = 0.f, Z = 0.f;
#pragma unroll
      for (int w = 0; w < NW_BF16; ++w) {
        const float f = (M == -INFINITY || mw[w] == -INFINITY) ? 0.f : ex2_approx(mw[w] - M);
        const float2 ov =
            *reinterpret_cast<const float2*>(&comb_o[(w * r + g) * RC_LD + col]);
        o0 = fmaf(ov.x, f, o0);
        o1 = fmaf(ov.y, f, o1);
        Z = fmaf(comb_z[w * GMAX + g], f, Z);
      }
      st_async_f32x2(dst + (uint32_t)(g * HD + col) * 4u, o0, o1, gbar);
      if (col == 0) st_async_f32x2(dst + (uint32_t)(r * HD + 2 * g) * 4u, M, Z, gbar);
    }
    if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 5 << 8);
    if (rank == 0) {
      // ----------------------------------------------- merge (CTA rank 0)
      // every CTA sends its slot whatever happened to its waits, so the
      // phase completes: after a failed wait, drain it before leaving (the
      // other CTAs' stores must not land in an exited CTA)
      if (!mbar_wait_cluster_bounded(&sm.gather_bar, 0u, abort_flag, p.wait_limit))
        mbar_drain_cluster(&sm.gather_bar, 0u);
      if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 6 << 8);
      bool waited = false;
      for (int pr = ct; pr < r * (HD / 2); pr += NT_BF16) {
        const int g = pr / (HD / 2), col = 2 * (pr % (HD / 2));
        const float2 o = CS <= 8 ? rc_merge_pair<8>(gather, slot, CS, r, g, col)
                                 : rc_merge_pair<16>(gather, slot, CS, r, g, col);
        if (!waited) {
          if (ct == 0) HYLRA_TRACE_CTA(tn, tcta, 11 << 8);
          griddep_wait();  // the preceding kernel has completed before out is written
          waited = true;
        }
        *reinterpret_cast<float2*>(p.out + ((size_t)b * p.Hq + (size_t)h * r + g) * HD + col) = o;
      }
    }
  }
  if (tid == 32) {
    HYLRA_TRACE_CTA(tn, tcta, 9 << 8);
    HYLRA_TRACE_VAL(tn, tcta, 42 << 8, HYLRA_CLOCK());
  }
  if (*abort_flag && tid == 32) atomicOr(p.status, HYLRA_STATUS_TIMEOUT);
}

// ------------------------------------------------------------ block gather
//
// Index-guided offloading (HyLRA summary §2.4): a reuse layer whose cache is
// in host memory needs only the blocks its index list names.  CTA (bh, e)
// copies block topk_in[b][h][e] of K and of V (the valid rows of it) from
// the host-resident cache (p.K, p.V: pinned host memory, read by the device
// across the host link) into slot e of the device staging cache
// [B][Hkv][k][128][d] (Ks, Vs).  Every thread keeps its loads in flight
// before storing, so the link sees many outstanding requests.
constexpr int NT_GATHER = 256;

__global__ void __launch_bounds__(NT_GATHER) gather_blocks_kernel(const __grid_constant__ Params p,
                                                                 uint8_t* Ks, uint8_t* Vs) {
  const int bh = (int)blockIdx.x, e = (int)blockIdx.y;  // B*Hkv may exceed a y extent
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int seqlen = valid_seqlen(p, b, false);
  const int nb = (seqlen + BLK - 1) / BLK;
  griddep_wait();  // the index list and the cache rows come from earlier work
  griddep_launch_dependents();
  if (e >= min(p.k, nb)) return;
  const int blk = __ldcg(p.topk_in + (size_t)bh * p.k + e);
  if (blk < 0 || blk >= nb) return;  // flagged by the reuse kernel
  if (p.newest_only && blk != nb - 1) return;
  const int rows = min(BLK, seqlen - blk * BLK);
  const long long src_row = row_base(p, b, h) + (long long)blk * BLK;
  const long long dst_row = ((long long)bh * p.k + e) * BLK;
  constexpr int CH = HD * 2 / 16;        // 16-byte chunks per row
  constexpr int PER = BLK * CH / NT_GATHER;  // chunks per thread and tensor
  const uint4* sk = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.K) + src_row * HD * 2);
  const uint4* sv = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.V) + src_row * HD * 2);
  uint4* dk = reinterpret_cast<uint4*>(Ks + dst_row * HD * 2);
  uint4* dv = reinterpret_cast<uint4*>(Vs + dst_row * HD * 2);
  uint4 vk[PER], vv[PER];
  const int nch = rows * CH;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int c = u * NT_GATHER + (int)threadIdx.x;
    if (c < nch) {
      vk[u] = sk[c];
      vv[u] = sv[c];
    }
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int c = u * NT_GATHER + (int)threadIdx.x;
    if (c < nch) {
      dk[c] = vk[u];
      dv[c] = vv[u];
    }
  }
}

// ------------------------------------------------ token-level profiling
//
// A profiling run may record top-k *token* indices instead of blocks (HyLRA
// summary §2.2 speaks of top-k token indices).  After a reset layer
// (decode_bf16_kernel<true> / decode_f32_kernel<true> + merge) the workspace
// holds every block's record (its max and its sum relative to it, per
// q-head).  head_stats_kernel reduces them to each head's max M_g and sum Z_g
// (log2 domain) and token_scores_kernel recomputes every token's logits and
// writes its attention mass summed over the group,
// score[t] = sum_g 2^(x_gt - M_g) / Z_g.  CUDA cores: this is profiling, not
// the decode path.
constexpr int NT_TOKEN = 128;  // one token per thread, one block per CTA

// Per (b, h): (M_g, Z_g) of its r heads into stats[bh][g] (float2).
__global__ void __launch_bounds__(NT_TOKEN) head_stats_kernel(const __grid_constant__ Params p,
                                                             float2* stats) {
  __shared__ float red_m[NT_TOKEN / 32][GMAX], red_z[NT_TOKEN / 32][GMAX];
  const int bh = (int)blockIdx.x, b = bh / p.Hkv;
  const int tid = (int)threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nb = (valid_seqlen(p, b, false) + BLK - 1) / BLK;
  for (int g = 0; g < p.r; ++g) {
    float M = -INFINITY, Z = 0.f;
    for (int beta = tid; beta < nb; beta += NT_TOKEN) {
      const float2 rec = *reinterpret_cast<const float2*>(p.bstat + bstat_at(p, bh, g, beta));
      if (rec.y == -INFINITY) continue;  // a block without valid tokens
      if (rec.y > M) {
        Z = Z * (M == -INFINITY ? 0.f : exp2f(M - rec.y));
        M = rec.y;
      }
      Z += rec.x * exp2f(rec.y - M);
    }
    // warp then CTA merge of (M, Z)
    for (int off = 16; off > 0; off >>= 1) {
      const float Mo = __shfl_xor_sync(0xffffffffu, M, off);
      const float Zo = __shfl_xor_sync(0xffffffffu, Z, off);
      const float Mn = fmaxf(M, Mo);
      Z = (Mn == -INFINITY) ? 0.f
                            : (M == -INFINITY ? 0.f : Z * exp2f(M - Mn)) +
                                  (Mo == -INFINITY ? 0.f : Zo * exp2f(Mo - Mn));
      M = Mn;
    }
    if (lane == 0) {
      red_m[wid][g] = M;
      red_z[wid][g] = Z;
    }
  }
  __syncthreads();
  if (tid < p.r) {
    const int g = tid;
    float M = -INFINITY;
    for (int w = 0; w < NT_TOKEN / 32; ++w) M = fmaxf(M, red_m[w][g]);
    float Z = 0.f;
    if (M != -INFINITY)
      for (int w = 0; w < NT_TOKEN / 32; ++w)
        if (red_m[w][g] != -INFINITY) Z += red_z[w][g] * exp2f(red_m[w][g] - M);
    stats[(size_t)bh * GMAX + g] = make_float2(M, Z);
  }
}

// Grid (nbmax, B * Hkv): token t = 128 * blockIdx.x + threadIdx.x of (b, h);
// scores [B][Hkv][max_seqlen], 0 past the sequence end.
template <typename T>
__global__ void __launch_bounds__(NT_TOKEN) token_scores_kernel(const __grid_constant__ Params p,
                                                               const float2* stats,
                                                               float* scores) {
  __shared__ float qs[GMAX][HD];
  __shared__ float2 st[GMAX];
  const int bh = (int)blockIdx.y, b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int tid = (int)threadIdx.x;
  const int n = valid_seqlen(p, b, false);
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)h * p.r) * HD;
  for (int e = tid; e < p.r * HD; e += NT_TOKEN) qs[e / HD][e % HD] = (float)qg[e];
  if (tid < p.r) st[tid] = stats[(size_t)bh * GMAX + tid];
  __syncthreads();
  const int t = (int)blockIdx.x * BLK + tid;
  if (t >= p.max_seqlen) return;
  float score = 0.f;
  if (t < n) {
    const T* krow = static_cast<const T*>(p.K) + (row_base(p, b, h) + t) * HD;
    float acc[GMAX];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) acc[g] = 0.f;
    for (int d = 0; d < HD; ++d) {
      const float kv = (float)krow[d];
#pragma unroll
      for (int g = 0; g < GMAX; ++g)
        if (g < p.r) acc[g] = fmaf(kv, qs[g][d], acc[g]);
    }
#pragma unroll
    for (int g = 0; g < GMAX; ++g)
      if (g < p.r && st[g].y > 0.f) score += exp2f(acc[g] * p.scale_log2 - st[g].x) / st[g].y;
  }
  scores[(size_t)bh * p.max_seqlen + t] = score;
}

// ------------------------------------------------------------ fp32 kernel

template <bool FULL>
__global__ void __launch_bounds__(NT_F32, 1) decode_f32_kernel(const __grid_constant__ Params p) {
  __shared__ SmemF32 sm;
  SmemCommon& c = sm.c;
  const int ct = threadIdx.x, cw = ct >> 5, lane = ct & 31;
  if (ct == 0) {
    c.nseg = 0;
    c.trace_n = 0;
    c.trace_cta = (int)blockIdx.x;
  }
  build_prefix(p, c, FULL);
  __syncthreads();
  const int T = c.prefix[p.B];
  const int G = T > 0 ? min((int)gridDim.x, T) : 1;
  const bool works = (int)blockIdx.x < G;
  const int lo = works ? (int)((long long)blockIdx.x * T / G) : 0;
  const int hi = works ? (int)((long long)(blockIdx.x + 1) * T / G) : 0;
  const int n = hi - lo;
  write_empty_outputs<FULL>(p, c);
  if (n <= 0) return;
  griddep_wait();  // the CUDA-core path is for small cases: no early start
  griddep_launch_dependents();

  const float* Kf = static_cast<const float*>(p.K);
  const float* Vf = static_cast<const float*>(p.V);
  float o[GMAX][4], m_run[GMAX], z_run[GMAX];
  UnitIter it;
  it.seek(c, p, lo);
  for (int i = 0; i < n; ++i) {
    const int blk_raw = FULL ? it.j : unit_index_entry(p, it);
    const StageMeta m = describe_unit<FULL>(p, c, it, i, n, T, G, valid_seqlen(p, it.b, false),
                                            blk_raw, ct == 0);
    it.advance(c, p);
    if (m.flags & F_SEG_START) {
      const float* qg = static_cast<const float*>(p.q) + ((size_t)m.b * p.Hq + (size_t)m.h * p.r) * HD;
      for (int e = ct; e < p.r * HD; e += NT_F32) sm.qs[e / HD][e % HD] = qg[e];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        m_run[g] = -INFINITY;
        z_run[g] = 0.f;
        o[g][0] = o[g][1] = o[g][2] = o[g][3] = 0.f;
      }
      named_bar_sync(BAR_CONS, NT_F32);
    }
    if (m.blk >= 0) {
      const long long row0 = row_base(p, m.b, m.h) + (long long)m.blk * BLK + cw * 32;
      const int t = cw * 32 + lane;
      const bool valid = t < m.nvalid;
      float acc[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) acc[g] = 0.f;
      if (valid) {
        const float4* kr = reinterpret_cast<const float4*>(Kf + (size_t)(row0 + lane) * HD);
        for (int d4 = 0; d4 < HD / 4; ++d4) {
          const float4 kv = kr[d4];
#pragma unroll
          for (int g = 0; g < GMAX; ++g) {
            if (g < p.r) {
              acc[g] = fmaf(kv.x, sm.qs[g][4 * d4], acc[g]);
              acc[g] = fmaf(kv.y, sm.qs[g][4 * d4 + 1], acc[g]);
              acc[g] = fmaf(kv.z, sm.qs[g][4 * d4 + 2], acc[g]);
              acc[g] = fmaf(kv.w, sm.qs[g][4 * d4 + 3], acc[g]);
            }
          }
        }
      }
      float pr[GMAX];
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g >= p.r) {
          pr[g] = 0.f;
          continue;
        }
        const float xg = valid ? acc[g] * p.scale_log2 : -INFINITY;
        float mx = xg;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float ms = mx == -INFINITY ? 0.f : mx;
        const float pv = ex2_approx(xg - ms);
        float sum = pv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (FULL && lane == 0) {
          sm.bst_s[i & 1][cw][g] = sum;
          sm.bst_m[i & 1][cw][g] = mx;
        }
        const float mn = fmaxf(m_run[g], mx);
        float al = 1.f, b = 0.f;
        if (mn != -INFINITY) {
          al = ex2_approx(m_run[g] - mn);
          b = ex2_approx(mx - mn);
        }
        z_run[g] = z_run[g] * al + sum * b;
        m_run[g] = mn;
        o[g][0] *= al;
        o[g][1] *= al;
        o[g][2] *= al;
        o[g][3] *= al;
        pr[g] = pv * b;
      }
      const int nv = max(0, min(32, m.nvalid - cw * 32));
      for (int tt = 0; tt < nv; ++tt) {
        const float4 v = reinterpret_cast<const float4*>(Vf + (size_t)(row0 + tt) * HD)[lane];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          if (g < p.r) {
            const float pt = __shfl_sync(0xffffffffu, pr[g], tt);
            o[g][0] = fmaf(pt, v.x, o[g][0]);
            o[g][1] = fmaf(pt, v.y, o[g][1]);
            o[g][2] = fmaf(pt, v.z, o[g][2]);
            o[g][3] = fmaf(pt, v.w, o[g][3]);
          }
        }
      }
    }
    if (FULL && m.blk >= 0) {
      named_bar_sync(BAR_CONS, NT_F32);
      if (cw == 0 && lane < p.r && meta_sane(p, m)) {
        float* dst = p.bstat + bstat_at(p, m.b * p.Hkv + m.h, lane, m.blk);
        float rec[2];
        combine_block_record<NW_F32>(sm.bst_s[i & 1], sm.bst_m[i & 1], lane, rec);
        dst[0] = rec[0];
        dst[1] = rec[1];
      }
    }
    if (m.flags & F_SEG_END) {
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        if (g < p.r) {
          c.comb_o[cw][g][lane * 4 + 0] = o[g][0];
          c.comb_o[cw][g][lane * 4 + 1] = o[g][1];
          c.comb_o[cw][g][lane * 4 + 2] = o[g][2];
          c.comb_o[cw][g][lane * 4 + 3] = o[g][3];
          if (lane == 0) {
            c.comb_m[cw][g] = m_run[g];
            c.comb_z[cw][g] = z_run[g];
          }
        }
      }
      named_bar_sync(BAR_CONS, NT_F32);
      store_partial<NT_F32, true>(p, c, m, ct);
      if (c.nseg == MAX_SEGS) flush_segments<FULL, NT_F32>(p, c, ct);
    }
  }
  flush_segments<FULL, NT_F32>(p, c, ct);
}

}  // namespace hylra
