// hylra_api.cu - C ABI entry points of the decode kernels (see include/hylra.h).
//
// Host side only: argument validation, workspace layout, TMA descriptor
// encoding and kernel launches.  The kernels live in hylra_kernels.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <mutex>
#include <vector>

#include "hylra.h"
#include "hylra_kernels.cuh"

using namespace hylra;

namespace {

constexpr size_t kSmemBF16 = sizeof(SmemBF16) + 1024;  // + alignment slack
constexpr int LATE_DEFICIT = 2;  // units fewer for streaming CTAs that start late
static_assert(kSmemBF16 <= 232448, "bf16 kernel shared memory exceeds 227 KB");
constexpr size_t kSmemMax = 232448;  // 227 KB of dynamic shared memory per CTA
static_assert(rc_smem_bytes(1, HYLRA_MAX_GROUP, 1) + 1024 <= kSmemMax,
              "cluster reuse kernel needs room for one stage");

struct Layout {
  size_t status, tickets, partials, bstat, total;
  int G, nbmax, nbh, nslots;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sm_count(int* G) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYLRA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  *G = std::min(n, MAX_CTAS);
  return HYLRA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(const hylra_shape_t* s) {
  if (!s) return HYLRA_ERR_INVALID;
  if (s->head_dim != HYLRA_HEAD_DIM || s->block_size != HYLRA_BLOCK_TOKENS)
    return HYLRA_ERR_UNSUPPORTED;
  if (s->batch < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1) return HYLRA_ERR_INVALID;
  if (s->num_q_heads % s->num_kv_heads != 0) return HYLRA_ERR_INVALID;
  if (s->num_q_heads / s->num_kv_heads > HYLRA_MAX_GROUP) return HYLRA_ERR_UNSUPPORTED;
  if (s->batch > HYLRA_MAX_BATCH) return HYLRA_ERR_UNSUPPORTED;
  if (s->topk < 1) return HYLRA_ERR_INVALID;
  if (s->topk > HYLRA_MAX_TOPK) return HYLRA_ERR_UNSUPPORTED;
  if (s->dtype != HYLRA_BF16 && s->dtype != HYLRA_FP32) return HYLRA_ERR_INVALID;
  if (s->max_seqlen < 0) return HYLRA_ERR_INVALID;
  if (s->max_seqlen > HYLRA_MAX_SEQLEN) return HYLRA_ERR_UNSUPPORTED;
  if (s->kv_capacity < 0) return HYLRA_ERR_INVALID;
  long long rows;
  if (s->kv_capacity > 0) {
    if (s->kv_capacity < s->max_seqlen) return HYLRA_ERR_INVALID;
    rows = (long long)s->batch * s->num_kv_heads * s->kv_capacity;
  } else {
    if (s->total_tokens < 0 || s->seq_offsets == nullptr) return HYLRA_ERR_INVALID;
    if (!aligned(s->seq_offsets, 8)) return HYLRA_ERR_INVALID;
    rows = (long long)s->num_kv_heads * s->total_tokens;
  }
  if (rows > INT_MAX - 2 * HYLRA_BLOCK_TOKENS) return HYLRA_ERR_UNSUPPORTED;
  const long long nbmax = (s->max_seqlen + HYLRA_BLOCK_TOKENS - 1) / HYLRA_BLOCK_TOKENS;
  if ((long long)s->batch * s->num_kv_heads * std::max(1LL, nbmax) > INT_MAX / 4)
    return HYLRA_ERR_UNSUPPORTED;
  return HYLRA_OK;
}

Layout make_layout(const hylra_shape_t* s, int G) {
  Layout L{};
  const int r = s->num_q_heads / s->num_kv_heads;
  L.G = G;
  L.nbmax = std::max(1, (s->max_seqlen + BLK - 1) / BLK);
  L.nbh = s->batch * s->num_kv_heads;
  L.nslots = G + L.nbh;
  size_t off = 0;
  L.status = off;
  off += 256;
  L.tickets = off;
  off = align_up(off + (size_t)L.nbh * 4, 256);
  L.partials = off;
  off = align_up(off + (size_t)L.nslots * SLOT_FLOATS * 4, 256);
  L.bstat = off;
  off = align_up(off + (size_t)L.nbh * L.nbmax * 2 * r * 4, 256);
  L.total = off;
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [rows][128] bf16 view with 64x128 boxes and 128-byte swizzle.
int make_tmap(CUtensorMap* tm, const void* base, long long rows) {
  auto fn = encode_fn();
  if (!fn) return HYLRA_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)HD, (cuuint64_t)std::max(1LL, rows)};
  cuuint64_t strides[1] = {(cuuint64_t)HD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BLK};
  cuuint32_t es[2] = {1, 1};
  const CUresult r =
      fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HYLRA_OK : HYLRA_ERR_CUDA;
}

// CTAs of the reset layers' merge kernel one SM holds at once (registers
// decide), per device; 1 if the query fails.
int merge_ctas_per_sm() {
  static std::mutex mu;
  static std::vector<int> cache;  // [dev]
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  int& v = cache[dev];
  if (v == 0) {
    int n = 0;
    const cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, merge_kernel, NT_MERGE, 0);
    if (e != cudaSuccess) cudaGetLastError();
    v = e == cudaSuccess ? std::max(1, n) : 1;
  }
  return v;
}

// Opt the bf16 kernels in to their dynamic shared memory once per device.
int prepare_bf16_kernels() {
  static std::mutex mu;
  static std::vector<char> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYLRA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)done.size() <= dev) done.resize(dev + 1, 0);
  if (done[dev]) return HYLRA_OK;
  if (cudaFuncSetAttribute(decode_bf16_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBF16) != cudaSuccess ||
      cudaFuncSetAttribute(decode_bf16_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBF16) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  done[dev] = 1;
  return HYLRA_OK;
}

// Cluster reuse kernel: cluster size (CTAs per (b, h)), blocks per CTA and
// pipeline stages.
struct RCPlan {
  int cs, upc, nst;
  bool comb_in_stage;
  size_t smem;
};

// Stages: one per block of the CTA up to NST_MAX_RC, as many as fit beside
// the gather area (0: this cluster size does not fit); when blocks outnumber
// the stages that fit, the warp states move into stage 0 at the end if that
// makes room for one more.
RCPlan rc_plan_for(int cs, int kmax, int r, int nst_cap = NST_MAX_RC) {
  RCPlan pl{};
  pl.cs = cs;
  pl.upc = (kmax + cs - 1) / cs;
  const int want = std::min(pl.upc, nst_cap);
  for (int alias = 0; alias < 2; ++alias) {
    const size_t fixed = rc_smem_bytes(cs, r, 0, alias != 0) + 1024;
    const int fit = fixed >= kSmemMax ? 0 : (int)((kSmemMax - fixed) / STAGE_BYTES);
    const int nst = std::min(want, fit);
    if (alias == 0 || nst > pl.nst) {
      pl.nst = nst;
      pl.comb_in_stage = alias != 0;
    }
    if (pl.nst >= want) break;
  }
  pl.smem = rc_smem_bytes(cs, r, pl.nst, pl.comb_in_stage) + 1024;
  return pl;
}

// Clusters of this shape the device can hold at once (queried once per
// device and shape).
int rc_max_active(const RCPlan& pl) {
  static std::mutex mu;
  static std::vector<std::vector<int>> cache;  // [dev][(cs * 4 + nst) * 64 + smem KB / 4]
  int dev = 0;
  if (pl.nst < 1 || pl.cs < 1 || pl.cs > 16) return 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, std::vector<int>(17 * 4 * 64, -1));
  int& v = cache[dev][(pl.cs * 4 + pl.nst) * 64 + (int)std::min<size_t>(63, pl.smem / 4096)];
  if (v < 0) {
    v = 0;
    if (cudaFuncSetAttribute(decode_reuse_cluster_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax) ==
            cudaSuccess &&
        cudaFuncSetAttribute(decode_reuse_cluster_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(pl.cs, 1);
      cfg.blockDim = dim3(NTHR_BF16);
      cfg.dynamicSmemBytes = pl.smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = pl.cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, decode_reuse_cluster_kernel, &cfg) == cudaSuccess)
        v = n;
    }
    cudaGetLastError();  // a refused query leaves no error behind
  }
  return v;
}

// Limit of the kernels' bounded waits, in SM clocks (hylra_set_wait_limit).
std::atomic<long long> g_wait_limit{WAIT_LIMIT_DEFAULT};

#if defined(HYLRA_TRACE) || defined(HYLRA_TUNE)
int g_plan_cs = 0, g_plan_nst = 0;  // tuning builds: force a plan
int g_late_deficit = -1;            // tuning builds: force the late-start deficit
#endif

// A small reuse layer (fewer blocks than SMs) is a latency chain: inside a
// decode step its CTAs are launched early and stage their blocks while the
// preceding layer runs, and after the wait each CTA computes its blocks and
// CTA 0 merges the cluster.  Two blocks per CTA, both staged, measured
// fastest on B200 (one block per CTA needs twice the clusters, of which
// fewer fit at once; three or more lengthen the chain after the wait).  A
// large layer spreads over every SM.
bool plan_reuse_cluster(const hylra_shape_t* s, RCPlan* out) {
  const int nbmax = std::max(1, (s->max_seqlen + BLK - 1) / BLK);
  const int kmax = std::max(1, std::min(s->topk, nbmax));
  const int nbh = s->batch * s->num_kv_heads;
  const int r = s->num_q_heads / s->num_kv_heads;
  if (nbh > 65535) return false;
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
#if defined(HYLRA_TRACE) || defined(HYLRA_TUNE)
  if (g_plan_cs < 0) return false;  // the stream-K split over every SM instead
  if (g_plan_cs > 0) {
    const RCPlan pl = rc_plan_for(std::min(g_plan_cs, kmax), kmax, r, g_plan_nst);
    if (pl.nst < 1 || rc_max_active(pl) < 1) return false;
    *out = pl;
    return true;
  }
#endif
  const bool small = (long long)nbh * kmax <= sms;
  if (small) {
    for (int cs = std::min(16, (kmax + 1) / 2); cs >= 1; --cs) {
      const RCPlan pl = rc_plan_for(cs, kmax, r);
      if (pl.nst >= 1 && rc_max_active(pl) >= nbh) {
        *out = pl;
        return true;
      }
    }
  }
  const int cs_max = std::max(1, std::min(std::min(16, kmax), sms / std::max(1, nbh)));
  for (int cs = cs_max; cs >= 1; --cs) {
    const RCPlan pl = rc_plan_for(cs, kmax, r);
    if (pl.nst < 1) continue;
    const int n = rc_max_active(pl);
    if (n >= nbh || (cs == 1 && n > 0)) {
      // A large layer (8 or more blocks per SM) whose clusters would leave
      // more than a tenth of the SMs idle (one CTA per SM) streams faster
      // over every SM with the cross-CTA merge kernel (B200: 8 x 64K and
      // the ragged 16-sequence batch, 3-6 % per reuse layer).
      if ((long long)nbh * kmax >= 8LL * sms && 10LL * pl.cs * nbh < 9LL * sms) return false;
      *out = pl;
      return true;
    }
  }
  return false;
}

int check_layer_ptrs(const hylra_shape_t* s, const void* q, const void* K, const void* V,
                     const float* out) {
  if (!q || !K || !V || !out) return HYLRA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16))
    return HYLRA_ERR_INVALID;
  (void)s;
  return HYLRA_OK;
}

// pdl: launch as a programmatic dependent of the preceding kernel in the
// stream (used between the layers of one decode step): the kernel's prologue
// and its K/V streaming may overlap the preceding kernel's tail; everything
// the preceding kernel writes is touched only after griddepcontrol.wait.
int launch(const hylra_shape_t* s, bool full, const void* q, const void* K, const void* V,
           const int32_t* seqlens, const int32_t* topk_in, float* out, int32_t* topk_out,
           void* ws, size_t ws_bytes, cudaStream_t stream, bool pdl = false,
           bool idx_from_prev = true, int trace_slot = 0, int late_ctas = 0,
           int* last_ctas = nullptr, bool staged = false) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (staged && (full || s->dtype != HYLRA_BF16)) return HYLRA_ERR_UNSUPPORTED;
  if ((rc = check_layer_ptrs(s, q, K, V, out))) return rc;
  if (!seqlens || !ws || !aligned(seqlens, 4) || !aligned(ws, 256)) return HYLRA_ERR_INVALID;
  if (full && (!topk_out || !aligned(topk_out, 4))) return HYLRA_ERR_INVALID;
  if (!full && (!topk_in || !aligned(topk_in, 4))) return HYLRA_ERR_INVALID;
  int G = 0;
  if ((rc = sm_count(&G))) return rc;
  const int G_sms = G;  // before G becomes this launch's streaming grid
  const Layout L = make_layout(s, G);
  if (ws_bytes < L.total) return HYLRA_ERR_WORKSPACE;

  uint8_t* w = static_cast<uint8_t*>(ws);
  Params p{};
  p.q = q;
  p.K = K;
  p.V = V;
  p.seqlens = seqlens;
  p.seq_off = s->kv_capacity > 0 ? nullptr : s->seq_offsets;
  p.topk_in = topk_in;
  p.out = out;
  p.topk_out = topk_out;
  p.status = reinterpret_cast<uint32_t*>(w + L.status);
  p.tickets = reinterpret_cast<uint32_t*>(w + L.tickets);
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.bstat = reinterpret_cast<float*>(w + L.bstat);
  p.cap = s->kv_capacity;
  p.total = s->kv_capacity > 0 ? 0 : s->total_tokens;
  p.B = s->batch;
  p.Hq = s->num_q_heads;
  p.Hkv = s->num_kv_heads;
  p.r = s->num_q_heads / s->num_kv_heads;
  p.k = s->topk;
  p.max_seqlen = s->max_seqlen;
  p.nbmax = L.nbmax;
  // a staged cache is written by the preceding kernel (the gather): wait
  // before any read, as for indices written just before
  p.idx_wait = (idx_from_prev || staged) ? 1 : 0;
  p.staged = staged ? 1 : 0;
  // CTAs launched early beside the preceding kernel stage their first blocks
  // before it ends; the last late_ctas of the grid (as many as the SMs the
  // preceding kernel holds) find their SMs still held
  // and start after it: they take LATE_DEFICIT units fewer (bf16 streaming)
  p.late_from = G - std::min(G, std::max(0, late_ctas));
  p.late_deficit = pdl && late_ctas > 0 ? LATE_DEFICIT : 0;
#if defined(HYLRA_TRACE) || defined(HYLRA_TUNE)
  if (g_late_deficit >= 0 && p.late_deficit > 0) p.late_deficit = g_late_deficit;
#endif
  if (last_ctas) *last_ctas = 0;
  p.q_wait = pdl ? 1 : 0;
  p.trace_slot = trace_slot;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);

  if (s->dtype == HYLRA_BF16) {
    if ((rc = prepare_bf16_kernels())) return rc;
    const long long rows =
        staged ? (long long)s->batch * s->num_kv_heads * s->topk * BLK
               : (s->kv_capacity > 0 ? (long long)s->batch * s->num_kv_heads * s->kv_capacity
                                     : (long long)s->num_kv_heads * s->total_tokens);
    CUtensorMap tmK, tmV;
    if ((rc = make_tmap(&tmK, K, rows))) return rc;
    if ((rc = make_tmap(&tmV, V, rows))) return rc;
    if (!full) {
      // reuse layers: one cluster per (b, h) when the device can schedule it
      const int nbh = s->batch * s->num_kv_heads;
      RCPlan pl{};
      if (plan_reuse_cluster(s, &pl)) {
        p.upc = pl.upc;
        p.nst = pl.nst;
        p.comb_in_stage = pl.comb_in_stage ? 1 : 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pl.cs, nbh);
        cfg.blockDim = dim3(NTHR_BF16);
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = pl.cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 2 : 1;
        if (cudaLaunchKernelEx(&cfg, decode_reuse_cluster_kernel, tmK, tmV, p) != cudaSuccess)
          return HYLRA_ERR_CUDA;
        if (last_ctas) *last_ctas = pl.cs * nbh;
        return cudaGetLastError() == cudaSuccess ? HYLRA_OK : HYLRA_ERR_CUDA;
      }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(NTHR_BF16);
    cfg.dynamicSmemBytes = kSmemBF16;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = full ? cudaLaunchKernelEx(&cfg, decode_bf16_kernel<true>, tmK, tmV, p)
                               : cudaLaunchKernelEx(&cfg, decode_bf16_kernel<false>, tmK, tmV, p);
    if (e != cudaSuccess) return HYLRA_ERR_CUDA;
    // the cross-CTA merge (and top-k) as the streaming kernel's dependent
    cudaLaunchConfig_t mcfg = {};
    // reset layers: per (b, h) a selection CTA and 1-4 output CTAs; reuse
    // layers: one small CTA per (b, h) (output merge and index-list check),
    // so that its CTAs hold few of the SMs the next layer's CTAs wait for
    const int nbh = s->batch * s->num_kv_heads;
    const int nout =
        full ? merge_out_ctas(s->num_q_heads / s->num_kv_heads, (long long)nbh, G_sms) : 0;
    mcfg.gridDim = dim3(nbh, 1 + nout);
    mcfg.blockDim = dim3(full ? NT_MERGE : NT_RMERGE);
    mcfg.dynamicSmemBytes = 0;
    mcfg.stream = stream;
    mcfg.attrs = attr;
    mcfg.numAttrs = 1;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    const cudaError_t em = full ? cudaLaunchKernelEx(&mcfg, merge_kernel, p, G)
                                : cudaLaunchKernelEx(&mcfg, merge_reuse_kernel, p, G);
    if (em != cudaSuccess) return HYLRA_ERR_CUDA;
    // SMs the merge kernel holds while the next layer's CTAs arrive (several
    // of its CTAs share an SM).  The reuse merge's CTAs could share an SM
    // five at a time, but they arrive as the streaming CTAs leave and spread
    // over the SMs freed first: a trace of the ragged16 step found its 128
    // CTAs on 42-57 SMs, so count three to an SM.
    if (last_ctas) {
      const int per_sm = full ? merge_ctas_per_sm() : 3;
      *last_ctas = std::min(G_sms, (nbh * (1 + nout) + per_sm - 1) / per_sm);
    }
  } else {
    if (full)
      decode_f32_kernel<true><<<G, NT_F32, 0, stream>>>(p);
    else
      decode_f32_kernel<false><<<G, NT_F32, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? HYLRA_OK : HYLRA_ERR_CUDA;
}

size_t elem_size(const hylra_shape_t* s) { return s->dtype == HYLRA_BF16 ? 2 : 4; }

size_t stage_bytes(const hylra_shape_t* s) {
  return (size_t)s->batch * s->num_kv_heads * s->topk * BLK * HD * 2;
}

int check_stage_rows(const hylra_shape_t* s) {
  const long long rows = (long long)s->batch * s->num_kv_heads * s->topk * BLK;
  return rows > INT_MAX - 2 * HYLRA_BLOCK_TOKENS ? HYLRA_ERR_UNSUPPORTED : HYLRA_OK;
}

// Copy the listed blocks of a host-resident cache into a staging cache.
int gather(const hylra_shape_t* s, const void* Kh, const void* Vh, const int32_t* seqlens,
           const int32_t* topk_in, void* Ks, void* Vs, cudaStream_t stream, bool pdl,
           bool newest_only = false) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (s->dtype != HYLRA_BF16) return HYLRA_ERR_UNSUPPORTED;
  if ((rc = check_stage_rows(s))) return rc;
  if (!Kh || !Vh || !seqlens || !topk_in || !Ks || !Vs) return HYLRA_ERR_INVALID;
  if (!aligned(Kh, 16) || !aligned(Vh, 16) || !aligned(Ks, 16) || !aligned(Vs, 16) ||
      !aligned(seqlens, 4) || !aligned(topk_in, 4))
    return HYLRA_ERR_INVALID;
  Params p{};
  p.K = Kh;
  p.V = Vh;
  p.seqlens = seqlens;
  p.seq_off = s->kv_capacity > 0 ? nullptr : s->seq_offsets;
  p.topk_in = topk_in;
  p.cap = s->kv_capacity;
  p.total = s->kv_capacity > 0 ? 0 : s->total_tokens;
  p.B = s->batch;
  p.Hq = s->num_q_heads;
  p.Hkv = s->num_kv_heads;
  p.r = s->num_q_heads / s->num_kv_heads;
  p.k = s->topk;
  p.max_seqlen = s->max_seqlen;
  // status bits of a bad length are left to the reuse kernel that follows
  p.status = nullptr;
  p.newest_only = newest_only ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s->batch * s->num_kv_heads, s->topk);
  cfg.blockDim = dim3(NT_GATHER);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, gather_blocks_kernel, p, static_cast<uint8_t*>(Ks),
                         static_cast<uint8_t*>(Vs)) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HYLRA_OK : HYLRA_ERR_CUDA;
}

// One decode step; offloaded (may be NULL): per layer, 1 = K[l], V[l] are a
// host-resident cache (reuse layers only), gathered into K_stage / V_stage.
// Host-side hooks around each layer's launches (stream order), used to
// interleave copies with the step; nullptr: none.
struct LayerHooks {
  int (*before)(void* ctx, int layer);
  int (*after)(void* ctx, int layer);
  void* ctx;
  // an offloaded reuse layer (index-guided offloading), given the layer of
  // the indices it reuses; sets *prev_ctas like launch()
  int (*offloaded)(void* ctx, int layer, int reset_layer, int* prev_ctas) = nullptr;
};

int run_step(const hylra_shape_t* shape, int32_t num_layers, const uint8_t* policy,
             const void* const* q, const void* const* K, const void* const* V,
             const uint8_t* offloaded, const int32_t* seqlens, float* const* out, int32_t* topk,
             void* K_stage, void* V_stage, void* workspace, size_t workspace_bytes,
             cudaStream_t stream, const LayerHooks* hooks = nullptr) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (num_layers < 1 || !policy || !q || !K || !V || !out || !topk) return HYLRA_ERR_INVALID;
  if (policy[0] != 1) return HYLRA_ERR_INVALID;
  for (int l = 0; l < num_layers; ++l) {
    if (policy[l] > 1) return HYLRA_ERR_INVALID;
    if (offloaded && offloaded[l] > 1) return HYLRA_ERR_INVALID;
    // a reset layer reads every block: its cache must be on the device
    if (offloaded && offloaded[l] && policy[l]) return HYLRA_ERR_INVALID;
    if ((rc = check_layer_ptrs(shape, q[l], K[l], V[l], out[l]))) return rc;
  }
  const size_t per_layer = (size_t)shape->batch * shape->num_kv_heads * shape->topk;
  int last_reset = 0;
  int prev_ctas = 0;  // SMs the kernel launched last holds (the next one's late CTAs)
  for (int l = 0; l < num_layers; ++l) {
    if (hooks && hooks->before && (rc = hooks->before(hooks->ctx, l))) return rc;
    if (policy[l]) {
      last_reset = l;
      rc = launch(shape, true, q[l], K[l], V[l], seqlens, nullptr, out[l], topk + l * per_layer,
                  workspace, workspace_bytes, stream, l > 0, true, l & 63, prev_ctas,
                  &prev_ctas);
    } else if (offloaded && offloaded[l]) {
      rc = hooks && hooks->offloaded ? hooks->offloaded(hooks->ctx, l, last_reset, &prev_ctas)
                                     : HYLRA_ERR_INVALID;
    } else {
      rc = launch(shape, false, q[l], K[l], V[l], seqlens, topk + last_reset * per_layer, out[l],
                  nullptr, workspace, workspace_bytes, stream, l > 0, last_reset == l - 1,
                  l & 63, prev_ctas, &prev_ctas);
    }
    if (rc) return rc;
    if (hooks && hooks->after && (rc = hooks->after(hooks->ctx, l))) return rc;
  }
  return HYLRA_OK;
}

// hylra_decode_step_host: a second stream carries the copies so that they
// overlap the step.  Layer 0's query goes first on the caller's stream, the
// other layers' queries on the copy stream (layer 1 waits for them), the
// outputs of every OUT_CHUNK layers go back as soon as those layers are done
// (towards the end in halving chunks, so that the copy left after the last
// layer is one layer's) and the indices once the last reset layer is; the
// caller's stream joins the copy stream at the end.
// The stream and events are per host thread and device.
constexpr int OUT_CHUNK = 8;

struct HostPipe {
  cudaStream_t main = nullptr, copy = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_q = nullptr, ev_out = nullptr, ev_join = nullptr;
  const uint8_t* q_host = nullptr;
  uint8_t* q_dev = nullptr;
  size_t q_layer_bytes = 0;
  const float* out_dev = nullptr;
  float* out_host = nullptr;
  size_t out_layer_floats = 0;
  const int32_t* topk_dev = nullptr;
  int32_t* topk_host = nullptr;
  size_t topk_layer = 0;
  int num_layers = 0, copied = 0;
  int last_reset = 0;  // the indices are final once this layer is done
};

int host_pipe_resources(HostPipe* hp) {
  struct Res {
    cudaStream_t copy = nullptr;
    cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
  };
  thread_local std::vector<Res> per_dev;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYLRA_ERR_CUDA;
  if ((int)per_dev.size() <= dev) per_dev.resize(dev + 1);
  Res& r = per_dev[dev];
  if (!r.copy) {
    if (cudaStreamCreateWithFlags(&r.copy, cudaStreamNonBlocking) != cudaSuccess) {
      r.copy = nullptr;
      return HYLRA_ERR_CUDA;
    }
    for (auto& e : r.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return HYLRA_ERR_CUDA;
  }
  hp->copy = r.copy;
  hp->ev_fork = r.ev[0];
  hp->ev_q = r.ev[1];
  hp->ev_out = r.ev[2];
  hp->ev_join = r.ev[3];
  return HYLRA_OK;
}

// After layer `done - 1`: the outputs of layers [copied, upto) back to the
// host and, once the last reset layer is done, all layers' indices (the
// step writes no others) in one copy.
int host_pipe_copy_out(HostPipe* hp, int upto, bool topk) {
  const bool out = upto > hp->copied && hp->out_host;
  topk = topk && hp->topk_host;
  if (!out && !topk) return HYLRA_OK;
  if (cudaEventRecord(hp->ev_out, hp->main) != cudaSuccess ||
      cudaStreamWaitEvent(hp->copy, hp->ev_out, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  if (topk && cudaMemcpyAsync(hp->topk_host, hp->topk_dev,
                              hp->num_layers * hp->topk_layer * sizeof(int32_t),
                              cudaMemcpyDeviceToHost, hp->copy) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  if (out) {
    const int l0 = hp->copied, n = upto - l0;
    if (cudaMemcpyAsync(hp->out_host + l0 * hp->out_layer_floats,
                        hp->out_dev + l0 * hp->out_layer_floats,
                        n * hp->out_layer_floats * sizeof(float), cudaMemcpyDeviceToHost,
                        hp->copy) != cudaSuccess)
      return HYLRA_ERR_CUDA;
    hp->copied = upto;
  }
  return HYLRA_OK;
}

int host_pipe_before(void* ctx, int layer) {
  HostPipe* hp = static_cast<HostPipe*>(ctx);
  // layer 1 on reads the queries that the copy stream brings in
  if (layer == 1 && cudaStreamWaitEvent(hp->main, hp->ev_q, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return HYLRA_OK;
}

int host_pipe_after(void* ctx, int layer) {
  HostPipe* hp = static_cast<HostPipe*>(ctx);
  const int done = layer + 1, left = hp->num_layers - done;
  // every OUT_CHUNK layers, and where the layers left halve below that
  const bool chunk = left > 0 && (done % OUT_CHUNK == 0 ||
                                  (left < OUT_CHUNK && (left & (left - 1)) == 0));
  if (chunk || layer == hp->last_reset)
    return host_pipe_copy_out(hp, chunk ? done : hp->copied, layer == hp->last_reset);
  return HYLRA_OK;
}



// Index-guided offloading with prefetch.  A second stream (one per host
// thread and device) gathers each offloaded layer's reused blocks from host
// memory into one of two staging slots as soon as the indices it reuses exist
// (its reset layer is done) and the slot is free (the layer that used it two
// offloaded layers earlier is done), so the link works while the layers run.
// The block holding each sequence's newest token is written by the preceding
// layer in a model: after that layer the caller's stream copies only those
// blocks again, then runs the reuse layer on the slot.
struct OffloadPipe {
  const hylra_shape_t* shape = nullptr;
  cudaStream_t main = nullptr, copy = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_reset = nullptr, ev_join = nullptr;
  cudaEvent_t ev_used[2] = {nullptr, nullptr}, ev_gathered[2] = {nullptr, nullptr};
  const uint8_t* policy = nullptr;
  const void* const* q = nullptr;
  const void* const* K = nullptr;
  const void* const* V = nullptr;
  const int32_t* seqlens = nullptr;
  float* const* out = nullptr;
  const int32_t* topk = nullptr;
  uint8_t* K_stage = nullptr;
  uint8_t* V_stage = nullptr;
  size_t slot_bytes = 0, per_layer = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<int> order;     // offloaded layers in order
  std::vector<int> pos_of;    // layer -> its place in `order` (-1: not offloaded)
  std::vector<int> reset_of;  // layer -> the reset layer whose indices it reuses
  int next = 0;               // next entry of `order` to gather
};

int offload_pipe_resources(OffloadPipe* op) {
  struct Res {
    cudaStream_t copy = nullptr;
    cudaEvent_t ev[7] = {};
  };
  thread_local std::vector<Res> per_dev;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYLRA_ERR_CUDA;
  if ((int)per_dev.size() <= dev) per_dev.resize(dev + 1);
  Res& r = per_dev[dev];
  if (!r.copy) {
    if (cudaStreamCreateWithFlags(&r.copy, cudaStreamNonBlocking) != cudaSuccess) {
      r.copy = nullptr;
      return HYLRA_ERR_CUDA;
    }
    for (auto& e : r.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return HYLRA_ERR_CUDA;
  }
  op->copy = r.copy;
  op->ev_fork = r.ev[0];
  op->ev_reset = r.ev[1];
  op->ev_join = r.ev[2];
  op->ev_used[0] = r.ev[3];
  op->ev_used[1] = r.ev[4];
  op->ev_gathered[0] = r.ev[5];
  op->ev_gathered[1] = r.ev[6];
  return HYLRA_OK;
}

// Gather every offloaded layer that can go now: layers < enq have been
// enqueued on the caller's stream.
int offload_pump(OffloadPipe* op, int enq) {
  while (op->next < (int)op->order.size()) {
    const int pos = op->next, j = op->order[pos], slot = pos & 1;
    const int i = op->reset_of[j];
    if (i >= enq) break;                                      // indices not enqueued yet
    if (pos >= 2 && op->order[pos - 2] >= enq) break;         // slot's last user not enqueued
    if (pos >= 2 && cudaStreamWaitEvent(op->copy, op->ev_used[slot], 0) != cudaSuccess)
      return HYLRA_ERR_CUDA;
    // ev_reset holds the record of reset layer i: a later reset would lie
    // between i and j, and j would reuse its indices instead
    if (cudaStreamWaitEvent(op->copy, op->ev_reset, 0) != cudaSuccess) return HYLRA_ERR_CUDA;
    int rc = gather(op->shape, op->K[j], op->V[j], op->seqlens, op->topk + i * op->per_layer,
                    op->K_stage + slot * op->slot_bytes, op->V_stage + slot * op->slot_bytes,
                    op->copy, false);
    if (rc) return rc;
    if (cudaEventRecord(op->ev_gathered[slot], op->copy) != cudaSuccess) return HYLRA_ERR_CUDA;
    ++op->next;
  }
  return HYLRA_OK;
}

int offload_before(void* ctx, int layer) { return offload_pump(static_cast<OffloadPipe*>(ctx), layer); }

int offload_after(void* ctx, int layer) {
  OffloadPipe* op = static_cast<OffloadPipe*>(ctx);
  if (op->policy[layer] && cudaEventRecord(op->ev_reset, op->main) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return offload_pump(op, layer + 1);
}

int offload_layer(void* ctx, int l, int reset_layer, int* prev_ctas) {
  OffloadPipe* op = static_cast<OffloadPipe*>(ctx);
  const int pos = op->pos_of[l], slot = pos & 1;
  if (pos < 0 || pos >= op->next) return HYLRA_ERR_INVALID;  // not gathered (cannot happen)
  const int32_t* idx = op->topk + reset_layer * op->per_layer;
  uint8_t* Ks = op->K_stage + slot * op->slot_bytes;
  uint8_t* Vs = op->V_stage + slot * op->slot_bytes;
  if (cudaStreamWaitEvent(op->main, op->ev_gathered[slot], 0) != cudaSuccess) return HYLRA_ERR_CUDA;
  // the newest token's block, after the preceding layer
  int rc = gather(op->shape, op->K[l], op->V[l], op->seqlens, idx, Ks, Vs, op->main, true, true);
  if (!rc)
    rc = launch(op->shape, false, op->q[l], Ks, Vs, op->seqlens, idx, op->out[l], nullptr, op->ws,
                op->ws_bytes, op->main, true, true, l & 63, 0, prev_ctas, true);
  if (rc) return rc;
  return cudaEventRecord(op->ev_used[slot], op->main) == cudaSuccess ? HYLRA_OK : HYLRA_ERR_CUDA;
}

}  // namespace

extern "C" {

int hylra_version(void) { return 100; }

const char* hylra_strerror(int err) {
  switch (err) {
    case HYLRA_OK: return "ok";
    case HYLRA_ERR_INVALID: return "invalid argument";
    case HYLRA_ERR_UNSUPPORTED: return "unsupported shape or limit exceeded";
    case HYLRA_ERR_CUDA: return "CUDA error";
    case HYLRA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown error";
  }
}

int hylra_workspace_bytes(const hylra_shape_t* shape, size_t* bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes) return HYLRA_ERR_INVALID;
  int G = 0;
  if ((rc = sm_count(&G))) return rc;
  *bytes = make_layout(shape, G).total;
  return HYLRA_OK;
}

int hylra_workspace_init(void* workspace, size_t bytes, hylra_stream_t stream) {
  if (!workspace) return HYLRA_ERR_INVALID;
  return cudaMemsetAsync(workspace, 0, bytes, (cudaStream_t)stream) == cudaSuccess
             ? HYLRA_OK
             : HYLRA_ERR_CUDA;
}

int hylra_decode_full(const hylra_shape_t* shape, const void* q, const void* K, const void* V,
                      const int32_t* seqlens, float* out, int32_t* topk_out, void* workspace,
                      size_t workspace_bytes, hylra_stream_t stream) {
  return launch(shape, true, q, K, V, seqlens, nullptr, out, topk_out, workspace,
                workspace_bytes, (cudaStream_t)stream);
}

int hylra_decode_reuse(const hylra_shape_t* shape, const void* q, const void* K, const void* V,
                       const int32_t* seqlens, const int32_t* topk_in, float* out,
                       void* workspace, size_t workspace_bytes, hylra_stream_t stream) {
  return launch(shape, false, q, K, V, seqlens, topk_in, out, nullptr, workspace,
                workspace_bytes, (cudaStream_t)stream);
}

int hylra_decode_step(const hylra_shape_t* shape, int32_t num_layers, const uint8_t* policy,
                      const void* const* q, const void* const* K, const void* const* V,
                      const int32_t* seqlens, float* const* out, int32_t* topk, void* workspace,
                      size_t workspace_bytes, hylra_stream_t stream) {
  return run_step(shape, num_layers, policy, q, K, V, nullptr, seqlens, out, topk, nullptr,
                  nullptr, workspace, workspace_bytes, (cudaStream_t)stream);
}

int hylra_token_scores(const hylra_shape_t* shape, const void* q, const void* K, const void* V,
                       const int32_t* seqlens, float* out, int32_t* topk_out, float* scores,
                       void* workspace, size_t workspace_bytes, hylra_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!scores || !aligned(scores, 4)) return HYLRA_ERR_INVALID;
  const int nbh = shape->batch * shape->num_kv_heads;
  const int nbmax = std::max(1, (shape->max_seqlen + BLK - 1) / BLK);
  if (nbh > 65535) return HYLRA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  // the reset layer itself: its block records stay in the workspace
  if ((rc = launch(shape, true, q, K, V, seqlens, nullptr, out, topk_out, workspace,
                   workspace_bytes, st)))
    return rc;
  int G = 0;
  if ((rc = sm_count(&G))) return rc;
  const Layout L = make_layout(shape, G);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  Params p{};
  p.q = q;
  p.K = K;
  p.V = V;
  p.seqlens = seqlens;
  p.seq_off = shape->kv_capacity > 0 ? nullptr : shape->seq_offsets;
  p.status = reinterpret_cast<uint32_t*>(w + L.status);
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.bstat = reinterpret_cast<float*>(w + L.bstat);
  p.cap = shape->kv_capacity;
  p.total = shape->kv_capacity > 0 ? 0 : shape->total_tokens;
  p.B = shape->batch;
  p.Hq = shape->num_q_heads;
  p.Hkv = shape->num_kv_heads;
  p.r = shape->num_q_heads / shape->num_kv_heads;
  p.k = shape->topk;
  p.max_seqlen = shape->max_seqlen;
  p.nbmax = L.nbmax;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  // the partials are consumed by the merge: their space holds the head statistics
  float2* stats = reinterpret_cast<float2*>(p.partials);
  head_stats_kernel<<<nbh, NT_TOKEN, 0, st>>>(p, stats);
  const dim3 grid(nbmax, nbh);
  if (shape->dtype == HYLRA_BF16)
    token_scores_kernel<__nv_bfloat16><<<grid, NT_TOKEN, 0, st>>>(p, stats, scores);
  else
    token_scores_kernel<float><<<grid, NT_TOKEN, 0, st>>>(p, stats, scores);
  return cudaGetLastError() == cudaSuccess ? HYLRA_OK : HYLRA_ERR_CUDA;
}

int hylra_stage_bytes(const hylra_shape_t* shape, size_t* bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes) return HYLRA_ERR_INVALID;
  if (shape->dtype != HYLRA_BF16) return HYLRA_ERR_UNSUPPORTED;
  if ((rc = check_stage_rows(shape))) return rc;
  *bytes = stage_bytes(shape);
  return HYLRA_OK;
}

int hylra_gather_blocks(const hylra_shape_t* shape, const void* K_host, const void* V_host,
                        const int32_t* seqlens, const int32_t* topk_in, void* K_stage,
                        void* V_stage, hylra_stream_t stream) {
  return gather(shape, K_host, V_host, seqlens, topk_in, K_stage, V_stage, (cudaStream_t)stream,
                false);
}

int hylra_decode_reuse_staged(const hylra_shape_t* shape, const void* q, const void* K_stage,
                              const void* V_stage, const int32_t* seqlens,
                              const int32_t* topk_in, float* out, void* workspace,
                              size_t workspace_bytes, hylra_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if ((rc = check_stage_rows(shape))) return rc;
  return launch(shape, false, q, K_stage, V_stage, seqlens, topk_in, out, nullptr, workspace,
                workspace_bytes, (cudaStream_t)stream, false, true, 0, 0, nullptr, true);
}

int hylra_decode_step_offload(const hylra_shape_t* shape, int32_t num_layers,
                              const uint8_t* policy, const void* const* q,
                              const void* const* K, const void* const* V,
                              const uint8_t* offloaded, const int32_t* seqlens,
                              float* const* out, int32_t* topk, void* K_stage, void* V_stage,
                              void* workspace, size_t workspace_bytes, hylra_stream_t stream) {
  if (!offloaded || !K_stage || !V_stage || !policy || !K || !V || num_layers < 1)
    return HYLRA_ERR_INVALID;
  int rc = check_shape(shape);
  if (rc) return rc;
  if (shape->dtype != HYLRA_BF16) return HYLRA_ERR_UNSUPPORTED;
  if ((rc = check_stage_rows(shape))) return rc;
  if (!aligned(K_stage, 16) || !aligned(V_stage, 16)) return HYLRA_ERR_INVALID;
  OffloadPipe op;
  if ((rc = offload_pipe_resources(&op))) return rc;
  op.shape = shape;
  op.main = (cudaStream_t)stream;
  op.policy = policy;
  op.q = q;
  op.K = K;
  op.V = V;
  op.seqlens = seqlens;
  op.out = out;
  op.topk = topk;
  op.K_stage = static_cast<uint8_t*>(K_stage);
  op.V_stage = static_cast<uint8_t*>(V_stage);
  op.slot_bytes = stage_bytes(shape);
  op.per_layer = (size_t)shape->batch * shape->num_kv_heads * shape->topk;
  op.ws = workspace;
  op.ws_bytes = workspace_bytes;
  op.pos_of.assign(num_layers, -1);
  op.reset_of.assign(num_layers, 0);
  for (int l = 0, last = 0; l < num_layers; ++l) {
    if (policy[l] == 1) last = l;
    op.reset_of[l] = last;
    if (offloaded[l] == 1 && policy[l] == 0) {
      op.pos_of[l] = (int)op.order.size();
      op.order.push_back(l);
    }
  }
  // the copy stream starts after the caller's earlier work and rejoins it
  if (cudaEventRecord(op.ev_fork, op.main) != cudaSuccess ||
      cudaStreamWaitEvent(op.copy, op.ev_fork, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  LayerHooks hooks{offload_before, offload_after, &op};
  hooks.offloaded = offload_layer;
  rc = run_step(shape, num_layers, policy, q, K, V, offloaded, seqlens, out, topk, K_stage,
                V_stage, workspace, workspace_bytes, op.main, &hooks);
  if (cudaEventRecord(op.ev_join, op.copy) != cudaSuccess ||
      cudaStreamWaitEvent(op.main, op.ev_join, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return rc;
}

int hylra_decode_step_host(const hylra_shape_t* shape, int32_t num_layers, const uint8_t* policy,
                           const void* q_host, void* q_dev, const void* const* K,
                           const void* const* V, const int32_t* seqlens, float* out_dev,
                           float* out_host, int32_t* topk_dev, int32_t* topk_host,
                           void* workspace, size_t workspace_bytes, hylra_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (num_layers < 1 || !q_host || !q_dev || !out_dev || !topk_dev || !K || !V)
    return HYLRA_ERR_INVALID;
  HostPipe hp;
  if ((rc = host_pipe_resources(&hp))) return rc;
  hp.main = (cudaStream_t)stream;
  const size_t q_layer = (size_t)shape->batch * shape->num_q_heads * HD;
  hp.q_host = static_cast<const uint8_t*>(q_host);
  hp.q_dev = static_cast<uint8_t*>(q_dev);
  hp.q_layer_bytes = q_layer * elem_size(shape);
  hp.out_dev = out_dev;
  hp.out_host = out_host;
  hp.out_layer_floats = q_layer;
  hp.topk_dev = topk_dev;
  hp.topk_host = topk_host;
  hp.topk_layer = (size_t)shape->batch * shape->num_kv_heads * shape->topk;
  hp.num_layers = num_layers;
  for (int l = 0; l < num_layers; ++l)
    if (policy && policy[l]) hp.last_reset = l;
  std::vector<const void*> qp(num_layers);
  std::vector<float*> op(num_layers);
  for (int l = 0; l < num_layers; ++l) {
    qp[l] = hp.q_dev + l * hp.q_layer_bytes;
    op[l] = out_dev + l * q_layer;
  }
  // layer 0's query on the caller's stream, the others on the copy stream
  if (cudaMemcpyAsync(hp.q_dev, hp.q_host, hp.q_layer_bytes, cudaMemcpyHostToDevice, hp.main) !=
          cudaSuccess ||
      cudaEventRecord(hp.ev_fork, hp.main) != cudaSuccess ||
      cudaStreamWaitEvent(hp.copy, hp.ev_fork, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  if (num_layers > 1 &&
      cudaMemcpyAsync(hp.q_dev + hp.q_layer_bytes, hp.q_host + hp.q_layer_bytes,
                      (num_layers - 1) * hp.q_layer_bytes, cudaMemcpyHostToDevice,
                      hp.copy) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  if (cudaEventRecord(hp.ev_q, hp.copy) != cudaSuccess) return HYLRA_ERR_CUDA;
  const LayerHooks hooks{host_pipe_before, host_pipe_after, &hp};
  rc = run_step(shape, num_layers, policy, qp.data(), K, V, nullptr, seqlens, op.data(), topk_dev,
                nullptr, nullptr, workspace, workspace_bytes, hp.main, &hooks);
  // the copy stream always rejoins the caller's stream (also after an error)
  const int rc_out = rc ? rc : host_pipe_copy_out(&hp, num_layers, false);
  if (cudaEventRecord(hp.ev_join, hp.copy) != cudaSuccess ||
      cudaStreamWaitEvent(hp.main, hp.ev_join, 0) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return rc_out;
}

#if defined(HYLRA_TRACE) || defined(HYLRA_TUNE)
// Tuning and trace builds only: force the reuse cluster plan (cs = 0: automatic,
// cs < 0: no cluster kernel).
int hylra_plan_override(int cs, int nst) {
  g_plan_cs = cs;
  g_plan_nst = nst;
  return HYLRA_OK;
}

int hylra_late_override(int d) {
  g_late_deficit = d;
  return HYLRA_OK;
}
#endif

#ifdef HYLRA_TRACE
// Trace builds only: device buffer of TRACE_PER_CTA uint64 per CTA (or NULL).
int hylra_trace_set(void* buf) {
  unsigned long long* p = static_cast<unsigned long long*>(buf);
  return cudaMemcpyToSymbol(g_hylra_trace, &p, sizeof(p)) == cudaSuccess ? HYLRA_OK
                                                                          : HYLRA_ERR_CUDA;
}
#endif

int hylra_set_wait_limit(int64_t cycles) {
  g_wait_limit.store(cycles > 0 ? (long long)cycles : WAIT_LIMIT_DEFAULT,
                     std::memory_order_relaxed);
  return HYLRA_OK;
}

int hylra_read_status(void* workspace, uint32_t* status, int clear, hylra_stream_t stream) {
  if (!workspace || !status) return HYLRA_ERR_INVALID;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HYLRA_ERR_CUDA;
  *status = v;
  if (clear && cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return HYLRA_OK;
}

// ------------------------------------------------ no-allocation entry point
//
// Some callers cannot hand the library a workspace: a serving process may
// reserve all free device memory for itself up front, cudaMalloc/cudaFree
// synchronise the device and are off limits inside latency-critical loops,
// and a thin foreign-language binding may have nowhere to keep a buffer
// alive between calls.  For them, hylra_decode_full_noalloc runs the reset
// layer kernel on a scratch area compiled into this library.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device

// Scratch of hylra_decode_full_noalloc.  It exists on every device that loads
// the library, for the life of the process.  In host code this name is only
// a host-side handle: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the first call on a device must not be inside a stream capture).
int noalloc_scratch(void** out) {
  static std::mutex mu;
  static std::vector<void*> addr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYLRA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)addr.size() <= dev) addr.resize(dev + 1, nullptr);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HYLRA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return HYLRA_OK;
}

}  // namespace

int hylra_decode_full_noalloc(const hylra_shape_t* shape, const void* q, const void* K,
                              const void* V, const int32_t* seqlens, float* out,
                              int32_t* topk_out, uint32_t* status_out, hylra_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  int G = 0;
  if ((rc = sm_count(&G))) return rc;
  const Layout L = make_layout(shape, G);
  if (L.total > kNoAllocScratchBytes) return HYLRA_ERR_WORKSPACE;  // shape too large for it
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // The scratch keeps whatever the previous call left: zero the status word
  // and the per-(sequence, KV head) tickets, which must start at zero.
  if (cudaMemsetAsync(scratch, 0, L.partials, st) != cudaSuccess) return HYLRA_ERR_CUDA;
  rc = hylra_decode_full(shape, q, K, V, seqlens, out, topk_out, scratch, kNoAllocScratchBytes,
                         stream);
  if (rc) return rc;
  if (status_out &&
      cudaMemcpyAsync(status_out, static_cast<unsigned char*>(scratch) + L.status,
                      sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return HYLRA_ERR_CUDA;
  return HYLRA_OK;
}

}  // extern "C"
