// pa_api.cu -- host side of libpagedattn: the C ABI declared in
// include/pagedattn.h, argument validation, and the dispatcher that picks the
// split-K partition size, kernel variant and grid.
//
// Dispatcher rule.  gllm PR #116 "feat(backend): sliding-window
// PagedAttention" ("What changes", CUDA): the launcher sizes its work from the
// longest *windowed* span, not the longest context.  ExecuTorch PR #18759
// (review suggestion 6) notes that a fixed 256-tokens-per-split rule ignores
// the SM count.  Here the partition size comes from the longest windowed span,
// the number of (row, kv head) units and the SMs x resident CTAs of the
// chosen kernel: few units get one balanced wave of partitions, many units
// get partitions of 2048..4096 tokens (about four waves where that fits).
// One partition per row means
// the one-shot path: the kernel writes dst itself, with no workspace and no
// reduce (aiter PR #2914 "Pa gluon swa mtp opt", one_shot).
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "../../include/pagedattn.h"
#include "pa_kernels.cuh"
#include "pa_span.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int succeed() {
  g_err.clear();
  return PA_OK;
}

constexpr int TS = pa::kStageTokens;
constexpr int kMinPartTokens = 256;
constexpr int kManyUnitsMinTokens = 2048;
constexpr int kManyUnitsMaxTokens = 4096;
constexpr int kPrefetchStages = 2;  // stages a one-wave CTA prefetches before its wait
constexpr unsigned long long kStageMaxBlocks = 512;  // CTAs per staging copy (256 threads each)

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_sms(int* out) {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return fail(PA_ERR_CUDA, "cannot read the SM count of device %d", dev);
    cache[dev] = n;
  }
  *out = cache[dev];
  return PA_OK;
}

int check_params(const pa_params* p, int bs) {
  if (!p) return fail(PA_ERR_ARG, "params is NULL");
  if (p->batch < 0 || p->batch > 65535)
    return fail(PA_ERR_ARG, "batch %d outside [0, 65535]", p->batch);
  if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_kv_heads > 65535)
    return fail(PA_ERR_ARG, "head counts must be positive (H_q=%d, H_kv=%d)", p->num_q_heads,
                p->num_kv_heads);
  if (p->num_q_heads % p->num_kv_heads != 0)
    return fail(PA_ERR_ARG, "H_q=%d is not a multiple of H_kv=%d", p->num_q_heads,
                p->num_kv_heads);
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d not supported (64, 128 or 256)", p->head_dim);
  if (!is_pow2(bs) || bs < 16 || bs > 1024)
    return fail(PA_ERR_UNSUPPORTED, "kvBlockSize %d not supported (power of two in [16,1024])", bs);
  if (p->num_blocks <= 0 || p->max_blocks_per_seq <= 0)
    return fail(PA_ERR_ARG, "num_blocks and max_blocks_per_seq must be positive");
  if ((long long)p->max_blocks_per_seq * bs > (long long)INT32_MAX)
    return fail(PA_ERR_ARG, "max_blocks_per_seq * kvBlockSize overflows int32");
  if (p->max_span_hint < 0 || p->max_query_len_hint < 0)
    return fail(PA_ERR_ARG, "hints must be >= 0");
  if (p->force_partitions < 0) return fail(PA_ERR_ARG, "force_partitions must be >= 0");
  if (p->wait_limit_cycles < 0 || p->merge_target_extra < 0)
    return fail(PA_ERR_ARG, "wait_limit_cycles and merge_target_extra must be >= 0");
  if (p->schedule != PA_SCHED_STATIC && p->schedule != PA_SCHED_WORKLIST)
    return fail(PA_ERR_ARG, "unknown schedule %d", p->schedule);
  if (p->force_variant != PA_VARIANT_AUTO && p->force_variant != PA_VARIANT_FMA &&
      p->force_variant != PA_VARIANT_MMA && p->force_variant != PA_VARIANT_TC)
    return fail(PA_ERR_ARG, "unknown force_variant %d", p->force_variant);
  // FP8 operands need their scales (aiter PR #2914 review: validate that
  // query_scale / key_scale / value_scale are present for FP8 tensors).
  auto good_scale = [](float x) { return x > 0.f && x <= 3.0e38f; };
  for (int dt : {p->q_dtype, p->kv_dtype})
    if (dt != PA_DTYPE_BF16 && dt != PA_DTYPE_FP8_E4M3)
      return fail(PA_ERR_ARG, "unknown dtype %d (q_dtype / kv_dtype)", dt);
  if (p->q_dtype == PA_DTYPE_FP8_E4M3 && !good_scale(p->q_scale))
    return fail(PA_ERR_ARG, "FP8 query needs a finite q_scale > 0 (got %g)", (double)p->q_scale);
  if (p->kv_dtype == PA_DTYPE_FP8_E4M3 && !(good_scale(p->k_scale) && good_scale(p->v_scale)))
    return fail(PA_ERR_ARG, "FP8 KV caches need finite k_scale and v_scale > 0 (got %g, %g)",
                (double)p->k_scale, (double)p->v_scale);
  return PA_OK;
}

bool any_fp8(const pa_params* p) {
  return p->q_dtype == PA_DTYPE_FP8_E4M3 || p->kv_dtype == PA_DTYPE_FP8_E4M3;
}

// Resident CTAs per SM of a kernel instance, queried once per device.
int cached_occupancy(bool mma, const pa::KernelShape& k, size_t smem) {
  // (k.tc selects the tensor-memory kernel)
  static std::mutex mu;
  static std::map<std::vector<long long>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const std::vector<long long> key = {dev, mma, k.head_dim, k.consumer_warps, k.stages, k.n8,
                                      k.kv_fp8, k.tc, (long long)smem};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int n = k.tc ? pa::occupancy_partition_tc(k, smem)
                : mma  ? pa::occupancy_partition_mma(k, smem)
                       : pa::occupancy_partition_fma(k, smem);
  if (n > 0) {
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = n;
  }
  return n;
}

struct Plan {
  pa_plan_info info;
  pa::KernelShape shape;
  size_t lse_bytes, o_bytes, ctr_bytes;
};

// span: longest union span over rows; qlen: longest queryLen.
int make_plan(const pa_params* p, int bs, int span, int qlen, int num_sms, int ctas_per_sm,
              Plan* out) {
  Plan pl;
  memset(&pl, 0, sizeof pl);
  const int G = p->num_q_heads / p->num_kv_heads;
  span = std::max(span, 1);
  qlen = std::max(qlen, 1);
  if ((long long)G * qlen > 4096)
    return fail(PA_ERR_UNSUPPORTED, "rows per kv head %lld exceed 4096", (long long)G * qlen);
  const int rmax = G * qlen;
  // Variant: the tensor-core kernel puts the KV tokens on the MMA's M axis
  // and the unit's rows on N (8 per tile), so it serves every row count; on
  // B200 it beats the CUDA-core FMA kernel even at 4 rows (GQA group 4 in an
  // 8-wide tile), because one m16n8k16 replaces ~40 FMA-path instructions per
  // token and the FMA kernel becomes issue-bound.  The FMA kernel stays for
  // pools whose row count exceeds the TMA map's 32-bit coordinates, and on
  // request.
  //
  // The tensor-memory kernel (FP8 caches, head_dim 128) runs on request: it
  // feeds the e4m3 codes to tcgen05 straight from shared memory, but its
  // softmax warps (one token per thread) spend more issue slots per token
  // than the conversions they save, so it trails the mma.sync kernel on the
  // named workloads.
  const bool rows_fit_tma =
      (long long)p->num_blocks * p->num_kv_heads * bs <= (long long)INT32_MAX;
  const bool kv8 = p->kv_dtype == PA_DTYPE_FP8_E4M3;
  const bool tc_shape = kv8 && p->head_dim == 128 && rows_fit_tma;
  int variant = p->force_variant;
  if (variant == PA_VARIANT_AUTO) variant = rows_fit_tma ? PA_VARIANT_MMA : PA_VARIANT_FMA;
  if (variant == PA_VARIANT_MMA && !rows_fit_tma)
    return fail(PA_ERR_UNSUPPORTED, "KV pool rows exceed the tensor map's 32-bit coordinates");
  if (variant == PA_VARIANT_TC && !tc_shape)
    return fail(PA_ERR_UNSUPPORTED,
                "the tensor-memory variant needs FP8 caches, head_dim 128 and a pool within the "
                "tensor map's 32-bit rows");
  const bool tc = variant == PA_VARIANT_TC;
  if (variant == PA_VARIANT_FMA && p->head_dim == 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim 256 runs on the tensor-core kernel only");
  if (variant == PA_VARIANT_FMA && any_fp8(p))
    return fail(PA_ERR_UNSUPPORTED, "FP8 operands run on the tensor-core kernel only");
  const bool mma = variant == PA_VARIANT_MMA || tc;  // TMA-staged kernels
  const int ncw = mma ? 4 : (rmax <= 16 ? 4 : 8);
  // tensor-core warps cover 8 rows (one n-tile) when the unit has <= 8 rows,
  // else 16 (head_dim 256: always 8, its accumulators are twice as wide); a
  // CTA covers up to 4 such tiles.
  const int n8 = (mma && !tc && rmax > 8 && p->head_dim <= 128) ? 2 : 1;
  pl.shape.n8 = n8;
  pl.shape.tc = tc;
  // the tensor-memory kernel covers 8 rows per CTA (its MMA's N is 16)
  const int slab_rows = tc ? 8 : mma ? 8 * n8 * ncw : 4 * ncw;
  const int nslab = (int)cdiv(rmax, slab_rows);
  pl.shape.head_dim = p->head_dim;
  pl.shape.consumer_warps = ncw;
  pl.shape.kv_fp8 = kv8;
  // bf16: 16, 32 or 64 KB per stage; FP8: 8, 16 or 32 KB per stage
  if (tc)
    pl.shape.stages = 3;  // 32 KB (128 tokens) per stage
  else if (!kv8)
    pl.shape.stages = p->head_dim == 64 ? 4 : 3;
  else
    pl.shape.stages = p->head_dim == 64 ? 8 : p->head_dim == 128 ? 4 : 3;

  // Partitions are whole stages: 64 tokens, 128 for the tensor-memory kernel.
  const int unit = tc ? 2 * TS : TS;
  // Partition-size cap: the CTA caches its slice of the block table in smem
  // (the tensor-memory kernel keeps it to 4096 tokens so two CTAs fit an SM).
  int cap = std::max(unit, ((pa::kMaxTableCache - 2) * bs) / unit * unit);
  if (tc) cap = std::min(cap, 4096);
  auto smem_for = [&](int ptok) {
    return tc    ? pa::tc_smem_bytes(pl.shape.stages, ptok, bs)
           : mma ? pa::mma_smem_bytes(p->head_dim, kv8 ? 1 : 2, pl.shape.stages, ptok, bs)
                 : pa::fma_smem_bytes(p->head_dim, pl.shape.stages, ptok, bs);
  };
  if (num_sms <= 0) {
    int rc = current_sms(&num_sms);
    if (rc) return rc;
  }
  const bool caller_occupancy = ctas_per_sm > 0;
  if (ctas_per_sm <= 0) {
    ctas_per_sm = cached_occupancy(mma, pl.shape, smem_for(cap));
    if (ctas_per_sm <= 0)
      return fail(PA_ERR_CUDA, "occupancy query failed: %s", cudaGetErrorString(cudaGetLastError()));
  }
  const long long units = (long long)p->batch * p->num_kv_heads * nslab;
  // FP8 caches, head_dim 128, units of one n-tile, a grid of few units (one
  // balanced wave): a six-stage ring at two CTAs per SM instead of four
  // stages at three.  Each CTA then has four stages in flight while its two
  // warp pairs work on the other two, and the wave has fewer, longer
  // partitions for the reduce to merge (faster on the long single-group
  // workload).  Grids of many units keep three CTAs per SM: there the extra
  // warps hide more latency than the deeper ring (it lost on GQA decode).
  if (kv8 && !tc && variant == PA_VARIANT_MMA && p->head_dim == 128 && n8 == 1 &&
      p->force_partitions <= 0 && !caller_occupancy) {
    pa::KernelShape deep = pl.shape;
    deep.stages = 6;
    const int c6 =
        cached_occupancy(true, deep, pa::mma_smem_bytes(p->head_dim, 1, 6, cap, bs));
    if (c6 > 0 && units * 4 <= (long long)num_sms * c6) {
      pl.shape = deep;
      ctas_per_sm = c6;
    }
  }
  const long long slots = (long long)num_sms * ctas_per_sm;

  long long ptok;
  if (p->force_partitions > 0) {
    ptok = cdiv(cdiv(span, p->force_partitions), unit) * unit;
  } else {
    if (units * 4 <= slots) {
      // few units: one balanced wave over every resident-CTA slot
      const long long want = std::max<long long>(1, cdiv(slots, std::max<long long>(units, 1)));
      ptok = std::max<long long>(cdiv(cdiv(span, want), unit) * unit, kMinPartTokens);
    } else {
      // many units: about four waves, but partitions of 2048..4096 tokens,
      // long enough to amortise a CTA's start-up and short enough that
      // ragged rows even out (measured on the named workloads)
      const long long want = std::max<long long>(1, cdiv(4 * slots, units));
      const long long target = std::min<long long>(
          std::max<long long>(cdiv(span, want), kManyUnitsMinTokens), kManyUnitsMaxTokens);
      // equal partitions: round the count to the nearest, so a row just over
      // a multiple of the target does not end in a sliver partition
      const long long aligned_span = (long long)span + TS - 1;
      const long long np = std::max<long long>(1, (aligned_span + target / 2) / target);
      ptok = cdiv(cdiv(aligned_span, np), unit) * unit;
    }
  }
  ptok = std::min<long long>(std::max<long long>(ptok, unit), cap);
  // At most 16384 partitions per row.
  ptok = std::max<long long>(ptok, cdiv(cdiv((long long)span + TS - 1, 16384), unit) * unit);
  const long long max_parts = cdiv((long long)span + TS - 1, ptok);
  if (max_parts > 16384) return fail(PA_ERR_UNSUPPORTED, "too many partitions");

  pa_plan_info& in = pl.info;
  in.variant = variant;
  in.partition_tokens = (int)ptok;
  in.max_partitions = (int)max_parts;
  in.one_shot = max_parts == 1;
  in.max_rows = rmax;
  in.slab_rows = slab_rows;
  in.consumer_warps = ncw;
  in.stages = pl.shape.stages;
  in.grid_x = (int)max_parts;
  in.grid_y = p->num_kv_heads * nslab;
  in.grid_z = p->batch;
  in.block_threads = tc ? 320 : 32 * (ncw + 1);
  in.smem_bytes = smem_for((int)ptok);
  in.num_sms = num_sms;
  in.ctas_per_sm = ctas_per_sm;
  if (p->schedule == PA_SCHED_WORKLIST) {
    const long long ctas = (long long)in.grid_x * in.grid_y * in.grid_z;
    if (variant != PA_VARIANT_MMA || ctas > slots)
      return fail(PA_ERR_UNSUPPORTED,
                  "the work-list schedule needs the MMA variant and a one-wave grid "
                  "(%lld CTAs, %lld slots)",
                  ctas, slots);
  }
  if (!in.one_shot) {
    const size_t partials = (size_t)p->batch * p->num_kv_heads * max_parts * rmax;
    pl.lse_bytes = align256(partials * sizeof(float));
    pl.o_bytes = align256(partials * p->head_dim * sizeof(float));
    in.worklist = p->schedule == PA_SCHED_WORKLIST;
    // two epoch-tagged counters per unit: stages handed out, partials published
    if (in.worklist)
      pl.ctr_bytes = align256(2 * (size_t)in.grid_z * in.grid_y * sizeof(uint64_t));
    in.workspace_bytes = pl.lse_bytes + pl.o_bytes + pl.ctr_bytes;
  }
  *out = pl;
  return PA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// The device address of a host buffer that kernels may read and write in
// place: pinned, mapped into the current context at the same address, with
// [p, p + bytes) inside one allocation.  nullptr for anything else (pageable
// or device memory, a range running past its allocation, a driver without the
// query), which the caller then moves with cudaMemcpyAsync.
void* mapped_host(const void* p, size_t bytes) {
  static PFN_cuPointerGetAttributes_v7000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuPointerGetAttributes", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuPointerGetAttributes_v7000>(f);
  });
  if (!fn || !p || bytes == 0) return nullptr;
  CUpointer_attribute at[5] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE, CU_POINTER_ATTRIBUTE_DEVICE_POINTER,
                               CU_POINTER_ATTRIBUTE_RANGE_START_ADDR,
                               CU_POINTER_ATTRIBUTE_RANGE_SIZE, CU_POINTER_ATTRIBUTE_MAPPED};
  // every slot is 8 bytes and zeroed: the driver writes 1 to 8 of them
  unsigned long long mtype = 0, dptr = 0, start = 0, size = 0, mapped = 0;
  void* data[5] = {&mtype, &dptr, &start, &size, &mapped};
  const CUdeviceptr addr = (CUdeviceptr)reinterpret_cast<uintptr_t>(p);
  if (fn(5, at, data, addr) != CUDA_SUCCESS) return nullptr;
  if ((unsigned int)mtype != CU_MEMORYTYPE_HOST || (mapped & 0xffu) == 0 || dptr != addr)
    return nullptr;
  if (addr < start || addr - start > size || bytes > size - (addr - start)) return nullptr;
  return reinterpret_cast<void*>(static_cast<uintptr_t>(dptr));
}

// One staging copy: the widest piece both addresses and the size allow.
pa::StageCopy stage_copy(const void* src, void* dst, size_t bytes) {
  const uintptr_t m = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | bytes;
  pa::StageCopy c;
  c.src = src;
  c.dst = dst;
  c.unit = (m & 15u) == 0 ? 16 : (m & 3u) == 0 ? 4 : 1;
  c.units = bytes / c.unit;
  c.first_block = 0;
  return c;
}

// 3-D map of a KV cache viewed as (box width W bytes, rows, row bytes / W
// sub-tiles), W = min(row bytes, 128): element stride 1, row stride
// head_dim * elem_bytes, sub-tile stride W bytes.  A box of (W, box_rows, all
// sub-tiles) lands in smem as [sub-tile][row][W bytes] with the W-byte
// swizzle (the sub-tile stride is smaller than the row stride on purpose: the
// box's sub-tiles become separate W-byte-wide tiles).  Encodings are cached
// per (base, rows, head_dim, elem_bytes, box_rows).
int kv_tensor_map(CUtensorMap* out, const void* base, long long rows, int head_dim,
                  int elem_bytes, int box_rows) {
  struct Entry {
    const void* base;
    long long rows;
    int d, eb, br;
    CUtensorMap map;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.base == base && e.rows == rows && e.d == head_dim && e.eb == elem_bytes &&
          e.br == box_rows) {
        *out = e.map;
        return PA_OK;
      }
  }
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const int row_bytes = head_dim * elem_bytes;
  const int w = std::min(row_bytes, 128);
  const cuuint64_t dims[3] = {(cuuint64_t)(w / elem_bytes), (cuuint64_t)rows,
                              (cuuint64_t)(row_bytes / w)};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)w};
  const cuuint32_t box[3] = {(cuuint32_t)(w / elem_bytes), (cuuint32_t)box_rows,
                             (cuuint32_t)(row_bytes / w)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  Entry e;
  e.base = base;
  e.rows = rows;
  e.d = head_dim;
  e.eb = elem_bytes;
  e.br = box_rows;
  const CUresult r = fn(&e.map,
                        elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        w == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 16) cache.erase(cache.begin());
  cache.push_back(e);
  *out = e.map;
  return PA_OK;
}

// Longest union span and query length from host copies of the lengths.
int host_extents(const int32_t* S, const int32_t* L, const int32_t* W, int window, int batch,
                 int* span, int* qlen, long long* ntok) {
  int sp = 0, ql = 0;
  long long nt = 0;
  for (int b = 0; b < batch; ++b) {
    const int w = W ? W[b] : window;
    if (L[b] < 0 || S[b] < 0 || L[b] > S[b] || w < 0)
      return fail(PA_ERR_ARG, "row %d: queryLen %d, seqLen %d, window %d are inconsistent", b, L[b],
                  S[b], w);
    nt += L[b];
    if (L[b] == 0) continue;
    sp = std::max(sp, pa::union_span(S[b], L[b], w));
    ql = std::max(ql, (int)L[b]);
  }
  *span = sp;
  *qlen = ql;
  if (ntok) *ntok = nt;
  return PA_OK;
}

int device_extents(const pa_params* p, const int32_t* seqLens, const int32_t* queryLens,
                   int window, cudaStream_t stream, int* span, int* qlen) {
  const int B = p->batch;
  std::vector<int32_t> S(B), L(B), W(p->windows ? B : 0);
  cudaError_t e = cudaMemcpyAsync(S.data(), seqLens, B * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(L.data(), queryLens, B * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess && p->windows)
    e = cudaMemcpyAsync(W.data(), p->windows, B * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reading lengths: %s", cudaGetErrorString(e));
  return host_extents(S.data(), L.data(), p->windows ? W.data() : nullptr, window, B, span, qlen,
                      nullptr);
}

int decode_impl(void* dst, const void* q, const void* kCache, const void* vCache,
                const int32_t* blockTables, const int32_t* seqLens, const int32_t* queryLens,
                float scale, int window, int bs, const pa_params* p, cudaStream_t stream,
                int span, int qlen) {
  Plan pl;
  int rc = make_plan(p, bs, span, qlen, 0, 0, &pl);
  if (rc) return rc;
  const pa_plan_info& in = pl.info;
  if (!in.one_shot) {
    if (!p->workspace || p->workspace_bytes < in.workspace_bytes)
      return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", in.workspace_bytes,
                  p->workspace ? p->workspace_bytes : (size_t)0);
    if (!aligned16(p->workspace)) return fail(PA_ERR_ARG, "workspace must be 16-byte aligned");
  }
  pa::DecodeArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.q8 = static_cast<const uint8_t*>(q);
  a.k_cache = kCache;
  a.v_cache = vCache;
  a.block_tables = blockTables;
  a.seq_lens = seqLens;
  a.query_lens = queryLens;
  a.windows = p->windows;
  a.dst = static_cast<__nv_bfloat16*>(dst);
  if (!in.one_shot) {
    char* ws = static_cast<char*>(p->workspace);
    a.ws_lse = reinterpret_cast<float*>(ws);
    a.ws_o = reinterpret_cast<float*>(ws + pl.lse_bytes);
    if (in.worklist) {
      // A graph replay would repeat the epoch recorded at capture, and a
      // replay's counters would then look current from the start.
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
        return fail(PA_ERR_UNSUPPORTED,
                    "the work-list schedule cannot be captured in a CUDA graph (per-call epoch)");
      static std::atomic<unsigned int> epochs{0};
      unsigned int e = ++epochs;
      if (e == 0) e = ++epochs;  // 0 is never a live epoch
      a.worklist = 1;
      a.epoch = e;
      a.stage_ctr = reinterpret_cast<unsigned long long*>(ws + pl.lse_bytes + pl.o_bytes);
      a.done = a.stage_ctr + (size_t)in.grid_z * in.grid_y;
    }
  }
  // FP8 scales: q_scale * k_scale multiplies every score, v_scale every output
  double sc = (double)scale * 1.4426950408889634;
  if (p->q_dtype == PA_DTYPE_FP8_E4M3) sc *= p->q_scale;
  if (p->kv_dtype == PA_DTYPE_FP8_E4M3) sc *= p->k_scale;
  a.scale_log2 = (float)sc;
  a.v_scale = p->kv_dtype == PA_DTYPE_FP8_E4M3 ? p->v_scale : 1.f;
  a.q_fp8 = p->q_dtype == PA_DTYPE_FP8_E4M3;
  a.window = window;
  a.batch = p->batch;
  a.num_q_heads = p->num_q_heads;
  a.num_kv_heads = p->num_kv_heads;
  a.group = p->num_q_heads / p->num_kv_heads;
  a.head_dim = p->head_dim;
  a.block_size = bs;
  a.block_shift = ilog2(bs);
  a.max_blocks_per_seq = p->max_blocks_per_seq;
  a.num_blocks = p->num_blocks;
  a.part_tokens = in.partition_tokens;
  a.max_parts = in.max_partitions;
  a.max_rows = in.max_rows;
  a.slab_rows = in.slab_rows;
  a.num_slabs = in.grid_y / p->num_kv_heads;
  a.wait_cycles = p->wait_limit_cycles > 0 ? p->wait_limit_cycles : pa::kWaitCycles;
  a.wait_extra = p->merge_target_extra > 0 ? (unsigned int)p->merge_target_extra : 0u;

  const dim3 grid(in.grid_x, in.grid_y, in.grid_z);
  // One wave of window-free partitions (the few-units plan): a CTA's first
  // copies need not wait for the lengths.  With many ragged rows (several
  // waves) the copies for empty partitions would cost more than they save.
  a.spec_first_stage = in.variant == PA_VARIANT_MMA && !in.worklist && !p->windows &&
                       window == 0 &&
                       (long long)in.grid_x * in.grid_y * in.grid_z <=
                           (long long)in.num_sms * in.ctas_per_sm;
  // Before their grid-dependency wait, these CTAs prefetch their first
  // stages into L2: in a decode loop the previous call's tail (its reduce,
  // the handoff) would otherwise leave HBM idle.  Two stages measured best on
  // the long single-group workload; three or more lost again (the prefetches
  // compete with the previous call's last loads).
  a.prefetch_stages = a.spec_first_stage ? kPrefetchStages : 0;
  a.prefetch_first = 0;
  // FP8 caches, units of at most 8 rows: the compute warps take the stages in
  // two pairs, two chunks at a time, and with the four-stage ring each warp
  // refills its own half stages (measured faster on the GQA decode and long
  // single-group workloads with FP8 caches).
  a.pair_chunks = in.variant == PA_VARIANT_MMA && p->kv_dtype == PA_DTYPE_FP8_E4M3 &&
                  in.max_rows <= 8 && !in.worklist;
  // Token rows per TMA box: a block, or a 64-token slice of a larger one; at
  // most 32 when the paired compute warps refill their own halves (the
  // four-stage FP8 ring), so that no box crosses a stage's halves.
  a.box_rows = std::min(bs, (a.pair_chunks && pl.shape.stages <= 4) ? TS / 2 : TS);
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  if (p->profile_events) {
    ev0 = static_cast<cudaEvent_t>(p->profile_events[0]);
    ev1 = static_cast<cudaEvent_t>(p->profile_events[1]);
  }
  cudaError_t e = ev0 ? cudaEventRecord(ev0, stream) : cudaSuccess;
  if (e == cudaSuccess) {
    if (in.variant == PA_VARIANT_MMA || in.variant == PA_VARIANT_TC) {
      CUtensorMap tk, tv;
      const long long rows = (long long)p->num_blocks * p->num_kv_heads * bs;
      const int br = in.variant == PA_VARIANT_TC ? std::min(bs, TS) : a.box_rows;
      const int eb = p->kv_dtype == PA_DTYPE_FP8_E4M3 ? 1 : 2;
      rc = kv_tensor_map(&tk, kCache, rows, p->head_dim, eb, br);
      if (!rc) rc = kv_tensor_map(&tv, vCache, rows, p->head_dim, eb, br);
      if (rc) return rc;
      e = in.variant == PA_VARIANT_TC
              ? pa::launch_partition_tc(a, pl.shape, tk, tv, grid, in.smem_bytes, stream)
              : pa::launch_partition_mma(a, pl.shape, tk, tv, grid, in.smem_bytes, stream);
    } else {
      e = pa::launch_partition_fma(a, pl.shape, grid, in.smem_bytes, stream);
    }
  }
  if (e == cudaSuccess && ev1) e = cudaEventRecord(ev1, stream);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "partition kernel launch: %s", cudaGetErrorString(e));
  if (!in.one_shot && !a.worklist) {
    e = pa::launch_reduce(a, stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reduce kernel launch: %s", cudaGetErrorString(e));
  }
  if (getenv("PA_LOG_PLAN"))
    fprintf(stderr,
            "[pagedattn] variant=%d ptok=%d parts=%d one_shot=%d rows=%d slab=%d warps=%d "
            "stages=%d grid=(%d,%d,%d) smem=%zu ws=%zu sms=%d ctas/sm=%d\n",
            in.variant, in.partition_tokens, in.max_partitions, in.one_shot, in.max_rows,
            in.slab_rows, in.consumer_warps, in.stages, in.grid_x, in.grid_y, in.grid_z,
            in.smem_bytes, in.workspace_bytes, in.num_sms, in.ctas_per_sm);
  return succeed();
}

}  // namespace

extern "C" {

int pa_decode(void* dst, const void* q, const void* kCache, const void* vCache,
              const int32_t* blockTables, const int32_t* seqLens, const int32_t* queryLens,
              float scale, int window, int kvBlockSize, const pa_params* params, void* stream) {
  int rc = check_params(params, kvBlockSize);
  if (rc) return rc;
  if (!dst || !q || !kCache || !vCache || !blockTables || !seqLens || !queryLens)
    return fail(PA_ERR_ARG, "a required pointer is NULL");
  if (!aligned16(dst) || !aligned16(q) || !aligned16(kCache) || !aligned16(vCache))
    return fail(PA_ERR_ARG, "dst, q, kCache and vCache must be 16-byte aligned");
  if (window < 0) return fail(PA_ERR_ARG, "window %d is negative", window);
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return fail(PA_ERR_ARG, "scale must be finite");
  if (params->batch == 0) return succeed();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int span = params->max_span_hint, qlen = params->max_query_len_hint;
  if (span == 0 || qlen == 0) {
    rc = device_extents(params, seqLens, queryLens, window, st, &span, &qlen);
    if (rc) return rc;
    if (qlen == 0) return succeed();  // every row has queryLen 0
  }
  return decode_impl(dst, q, kCache, vCache, blockTables, seqLens, queryLens, scale, window,
                     kvBlockSize, params, st, span, qlen);
}

size_t pa_workspace_size(const pa_params* params, int kvBlockSize) {
  if (check_params(params, kvBlockSize)) return (size_t)-1;
  const int span = params->max_span_hint > 0 ? params->max_span_hint
                                             : params->max_blocks_per_seq * kvBlockSize;
  const int qlen = params->max_query_len_hint > 0 ? params->max_query_len_hint : 1;
  Plan pl;
  if (make_plan(params, kvBlockSize, span, qlen, 0, 0, &pl)) return (size_t)-1;
  succeed();
  return pl.info.workspace_bytes;
}

int pa_plan(const pa_params* params, int kvBlockSize, int num_sms, int ctas_per_sm,
            pa_plan_info* out) {
  int rc = check_params(params, kvBlockSize);
  if (rc) return rc;
  if (!out) return fail(PA_ERR_ARG, "out is NULL");
  const int span = params->max_span_hint > 0 ? params->max_span_hint
                                             : params->max_blocks_per_seq * kvBlockSize;
  const int qlen = params->max_query_len_hint > 0 ? params->max_query_len_hint : 1;
  Plan pl;
  rc = make_plan(params, kvBlockSize, span, qlen, num_sms, ctas_per_sm, &pl);
  if (rc) return rc;
  *out = pl.info;
  return succeed();
}

int pa_visible_ranges(int32_t* lo, int32_t* hi, const int32_t* seqLens, const int32_t* queryLens,
                      int window, const int32_t* windows, int batch, void* stream) {
  if (!lo || !hi || !seqLens || !queryLens) return fail(PA_ERR_ARG, "a required pointer is NULL");
  if (batch < 0) return fail(PA_ERR_ARG, "batch %d is negative", batch);
  if (window < 0) return fail(PA_ERR_ARG, "window %d is negative", window);
  if (batch == 0) return succeed();
  cudaError_t e = pa::launch_ranges(lo, hi, seqLens, queryLens, window, windows, batch,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "ranges kernel launch: %s", cudaGetErrorString(e));
  return succeed();
}

int pa_unreachable_blocks(int32_t* count, const int32_t* seqLens, const int32_t* queryLens,
                          int window, const int32_t* windows, int kvBlockSize, int batch,
                          void* stream) {
  if (!count || !seqLens || !queryLens) return fail(PA_ERR_ARG, "a required pointer is NULL");
  if (batch < 0) return fail(PA_ERR_ARG, "batch %d is negative", batch);
  if (window < 0) return fail(PA_ERR_ARG, "window %d is negative", window);
  if (!is_pow2(kvBlockSize) || kvBlockSize < 16 || kvBlockSize > 1024)
    return fail(PA_ERR_UNSUPPORTED, "kvBlockSize %d not supported (power of two in [16,1024])",
                kvBlockSize);
  if (batch == 0) return succeed();
  cudaError_t e = pa::launch_unreachable(count, seqLens, queryLens, window, windows,
                                         ilog2(kvBlockSize), batch, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return succeed();
}

size_t pa_host_workspace_size(const pa_params* params, int kvBlockSize, int window,
                              const int32_t* seqLens_host, const int32_t* queryLens_host) {
  if (check_params(params, kvBlockSize) || !seqLens_host || !queryLens_host) return (size_t)-1;
  int span = 0, qlen = 0;
  long long ntok = 0;
  if (window < 0) return (size_t)-1;
  if (host_extents(seqLens_host, queryLens_host, params->windows, window, params->batch, &span,
                   &qlen, &ntok))
    return (size_t)-1;
  const size_t B = params->batch;
  const size_t rowe = (size_t)ntok * params->num_q_heads * params->head_dim;
  const size_t qbytes = align256(rowe * (params->q_dtype == PA_DTYPE_FP8_E4M3 ? 1 : 2));
  size_t total = qbytes + align256(rowe * 2) + align256(B * params->max_blocks_per_seq * 4) +
                 3 * align256(B * 4);
  if (qlen > 0) {
    Plan pl;
    if (make_plan(params, kvBlockSize, span, qlen, 0, 0, &pl)) return (size_t)-1;
    total += pl.info.workspace_bytes;
  }
  succeed();
  return total;
}

int pa_decode_host(void* dst_host, const void* q_host, const void* kCache, const void* vCache,
                   const int32_t* blockTables_host, const int32_t* seqLens_host,
                   const int32_t* queryLens_host, float scale, int window, int kvBlockSize,
                   const pa_params* params, void* stream) {
  int rc = check_params(params, kvBlockSize);
  if (rc) return rc;
  if (!dst_host || !q_host || !kCache || !vCache || !blockTables_host || !seqLens_host ||
      !queryLens_host)
    return fail(PA_ERR_ARG, "a required pointer is NULL");
  if (window < 0) return fail(PA_ERR_ARG, "window %d is negative", window);
  if (!aligned16(kCache) || !aligned16(vCache))
    return fail(PA_ERR_ARG, "kCache and vCache must be 16-byte aligned");
  const int B = params->batch;
  if (B == 0) return succeed();
  int span = 0, qlen = 0;
  long long ntok = 0;
  rc = host_extents(seqLens_host, queryLens_host, params->windows, window, B, &span, &qlen, &ntok);
  if (rc) return rc;
  const size_t need =
      pa_host_workspace_size(params, kvBlockSize, window, seqLens_host, queryLens_host);
  if (need == (size_t)-1) return fail(PA_ERR_ARG, "%s", g_err.c_str());
  if (!params->workspace || params->workspace_bytes < need)
    return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                params->workspace ? params->workspace_bytes : (size_t)0);
  if (!aligned16(params->workspace)) return fail(PA_ERR_ARG, "workspace must be 16-byte aligned");

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(params->workspace);
  const size_t rowe = (size_t)ntok * params->num_q_heads * params->head_dim;
  const size_t qbytes_raw = rowe * (params->q_dtype == PA_DTYPE_FP8_E4M3 ? 1 : 2);
  const size_t dbytes_raw = rowe * 2;
  const size_t btbytes = (size_t)B * params->max_blocks_per_seq * 4;
  char* d_q = ws;
  char* d_dst = d_q + align256(qbytes_raw);
  char* d_bt = d_dst + align256(dbytes_raw);
  char* d_S = d_bt + align256(btbytes);
  char* d_L = d_S + align256((size_t)B * 4);
  char* d_W = d_L + align256((size_t)B * 4);
  char* d_split = d_W + align256((size_t)B * 4);

  // Inputs in.  Pinned host buffers that are mapped into this context are
  // read in place by one staging kernel (a DMA copy per buffer costs several
  // microseconds of fixed latency each); the others are copied.
  struct In {
    const void* src;
    void* dst;
    size_t bytes;
  } ins[5] = {{q_host, d_q, qbytes_raw},
              {blockTables_host, d_bt, btbytes},
              {seqLens_host, d_S, (size_t)B * 4},
              {queryLens_host, d_L, (size_t)B * 4},
              {params->windows, d_W, params->windows ? (size_t)B * 4 : 0}};
  pa::StageArgs sa;
  memset(&sa, 0, sizeof sa);
  cudaError_t e = cudaSuccess;
  for (const In& in : ins) {
    if (!in.bytes) continue;
    const void* mapped = mapped_host(in.src, in.bytes);
    if (mapped) {
      pa::StageCopy c = stage_copy(mapped, in.dst, in.bytes);
      c.first_block = sa.blocks;
      sa.blocks += (int)std::min<unsigned long long>((c.units + 255) / 256, kStageMaxBlocks);
      sa.c[sa.n++] = c;
    } else if (e == cudaSuccess) {
      e = cudaMemcpyAsync(in.dst, in.src, in.bytes, cudaMemcpyHostToDevice, st);
    }
  }
  if (e == cudaSuccess && sa.n) e = pa::launch_stage(sa, st);
  if (e != cudaSuccess) {
    cudaStreamSynchronize(st);  // copies already queued finish before the buffers go back
    return fail(PA_ERR_CUDA, "host-to-device copy: %s", cudaGetErrorString(e));
  }
  // Output: a mapped, 16-byte aligned dst is written by the kernels in place.
  void* dst_mapped = aligned16(dst_host) ? mapped_host(dst_host, dbytes_raw) : nullptr;
  if (dst_mapped) d_dst = static_cast<char*>(dst_mapped);

  if (qlen > 0) {
    pa_params dp = *params;
    dp.windows = params->windows ? reinterpret_cast<const int32_t*>(d_W) : nullptr;
    dp.workspace = d_split;
    dp.workspace_bytes = params->workspace_bytes - (size_t)(d_split - ws);
    dp.max_span_hint = span;
    dp.max_query_len_hint = qlen;
    rc = decode_impl(d_dst, d_q, kCache, vCache, reinterpret_cast<const int32_t*>(d_bt),
                     reinterpret_cast<const int32_t*>(d_S), reinterpret_cast<const int32_t*>(d_L),
                     scale, window, kvBlockSize, &dp, st, span, qlen);
    if (rc) {
      // the staging copies (and any kernel already launched) may still read
      // or write the caller's host buffers: let them finish before returning
      const std::string msg = g_err;
      cudaStreamSynchronize(st);
      g_err = msg;
      return rc;
    }
  }
  if (dbytes_raw && !dst_mapped)
    e = cudaMemcpyAsync(dst_host, d_dst, dbytes_raw, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "device-to-host copy: %s", cudaGetErrorString(e));
  return succeed();
}

int pa_extents_host(const int32_t* seqLens, const int32_t* queryLens, const int32_t* windows,
                    int window, int batch, int* max_span, int* max_query_len) {
  if (!seqLens || !queryLens || !max_span || !max_query_len)
    return fail(PA_ERR_ARG, "a required pointer is NULL");
  if (batch < 0 || window < 0) return fail(PA_ERR_ARG, "batch and window must be >= 0");
  int rc = host_extents(seqLens, queryLens, windows, window, batch, max_span, max_query_len, nullptr);
  if (rc) return rc;
  return succeed();
}

int pa_device_status(unsigned int* status, int clear, void* stream) {
  if (!status) return fail(PA_ERR_ARG, "status is NULL");
  cudaError_t e = pa::read_status(status, clear != 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reading status: %s", cudaGetErrorString(e));
  return succeed();
}

const char* pa_last_error(void) { return g_err.c_str(); }

const char* pa_version(void) { return "libpagedattn 0.1 (sm_100a)"; }

}  // extern "C"
