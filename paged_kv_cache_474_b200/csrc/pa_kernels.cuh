// pa_kernels.cuh -- launch interface between the host dispatcher (pa_api.cu)
// and the sm_100a kernels (pa_partition.cu, pa_reduce.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace pa {

constexpr int kStageTokens = 64;  // tokens per shared-memory pipeline stage
constexpr int kMaxTableCache = 1024;  // block-table entries a CTA caches in smem
// Limit of every bounded device wait, in SM clocks (about a second at the
// B200's clocks); the work-list merge's wait takes pa_params.wait_limit_cycles
// instead when that test knob is set.
constexpr long long kWaitCycles = 2000000000LL;

// Everything a decode launch needs; passed by value as a __grid_constant__.
struct DecodeArgs {
  const __nv_bfloat16* q;  // bf16 queries (q_fp8 == 0)
  const uint8_t* q8;       // FP8 e4m3 query codes (q_fp8 == 1)
  const void* k_cache;     // bf16, or FP8 e4m3 codes (tensor-core kernel only)
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const int32_t* query_lens;
  const int32_t* windows;  // may be null
  __nv_bfloat16* dst;
  float* ws_lse;  // [B][H_kv][max_parts][max_rows]  log2-domain lse of each partial
  float* ws_o;    // [B][H_kv][max_parts][max_rows][D] normalised partial outputs
  float scale_log2;  // scale * log2(e) (* q_scale * k_scale for FP8 operands): log2-domain scores
  float v_scale;     // multiplies every output (FP8 V), 1 otherwise
  int q_fp8;
  int window;
  int batch, num_q_heads, num_kv_heads, group, head_dim;
  int block_size, block_shift, max_blocks_per_seq, num_blocks;
  int part_tokens;  // tokens per partition, a multiple of kStageTokens
  int max_parts;    // partitions per unit the workspace holds (1 = one-shot)
  int max_rows;     // rows per unit the workspace holds
  int slab_rows;    // rows one CTA handles
  int num_slabs;    // CTAs per unit along grid.y (grid.y = H_kv * num_slabs)
  // One-wave grids of window-free rows: each CTA issues its partition's first
  // stage before the lengths arrive (the longest rows fill the grid, so few
  // of those copies are for partitions past a row's end).
  int spec_first_stage;
  // Stages of its partition each CTA prefetches into L2 before the
  // grid-dependency wait (0: none), for the same one-wave grids of window-free
  // rows: while the previous kernel drains, HBM would otherwise idle.
  int prefetch_stages;
  int prefetch_first;  // first stage of the partition it prefetches
  int box_rows;        // token rows per TMA box of the tensor-core kernel (<= 32 in paired mode)
  // Tensor-core kernel with FP8 caches, units of at most 8 rows: the compute
  // warps work in two pairs on alternating stages, two chunks at a time.
  int pair_chunks;
  // Work-list schedule (tensor-core kernel, one-wave cooperative grid): a
  // unit's CTAs claim its 64-token stages from a counter and merge their own
  // partials instead of a reduce kernel.
  int worklist;
  unsigned int epoch;             // this call's tag for the counters below
  unsigned long long* stage_ctr;  // [B][grid.y] next stage to hand out
  unsigned long long* done;       // [B][grid.y] partials published
  long long wait_cycles;          // limit of the merge's wait for arrivals (SM clocks)
  unsigned int wait_extra;        // test knob: arrivals added to that wait's target
};

// Compile-time shape of a partition-kernel instance.
struct KernelShape {
  int head_dim;
  int consumer_warps;
  int stages;
  int n8;  // tensor-core variant: 8-row n-tiles per compute warp (1 or 2)
  int kv_fp8;  // tensor-core variant: FP8 e4m3 K/V caches
  int tc;      // tensor-memory (tcgen05) variant
};

// Dynamic shared memory of the FMA partition kernel.
size_t fma_smem_bytes(int head_dim, int stages, int part_tokens, int block_size);

// Launches the FMA partition kernel; returns the launch error.
cudaError_t launch_partition_fma(const DecodeArgs& a, const KernelShape& k, dim3 grid,
                                 size_t smem, cudaStream_t stream);

// Occupancy (CTAs per SM) of an FMA partition-kernel instance.
int occupancy_partition_fma(const KernelShape& k, size_t smem);

// Dynamic shared memory of the tensor-core partition kernel.
size_t mma_smem_bytes(int head_dim, int elem_bytes, int stages, int part_tokens, int block_size);

// Launches the tensor-core partition kernel; tk / tv are 3-D tiled maps of
// the K and V caches: (box width, rows, row bytes / box width) with boxes of
// (box width, box rows, all) and the 128-byte swizzle (64-byte for the
// 64-byte rows of FP8 head_dim 64); box width = min(row bytes, 128) bytes.
cudaError_t launch_partition_mma(const DecodeArgs& a, const KernelShape& k, const CUtensorMap& tk,
                                 const CUtensorMap& tv, dim3 grid, size_t smem,
                                 cudaStream_t stream);
// (a.worklist launches cooperatively: every CTA of the grid is resident at once.)

int occupancy_partition_mma(const KernelShape& k, size_t smem);

// Dynamic shared memory of the tensor-memory (tcgen05) partition kernel
// (FP8 caches, head_dim 128, 128-token stages).
size_t tc_smem_bytes(int stages, int part_tokens, int block_size);

// Launches the tcgen05 partition kernel (320 threads); tk / tv as for the
// tensor-core kernel with FP8 caches.
cudaError_t launch_partition_tc(const DecodeArgs& a, const KernelShape& k, const CUtensorMap& tk,
                                const CUtensorMap& tv, dim3 grid, size_t smem,
                                cudaStream_t stream);

int occupancy_partition_tc(const KernelShape& k, size_t smem);

// Launches the log-sum-exp reduce over (rows, kv heads, batch).
cudaError_t launch_reduce(const DecodeArgs& a, cudaStream_t stream);

// Launches the visible-range kernel.
cudaError_t launch_ranges(int32_t* lo, int32_t* hi, const int32_t* seq_lens,
                          const int32_t* query_lens, int window, const int32_t* windows,
                          int batch, cudaStream_t stream);

// Launches the dead-leading-block count per row.
cudaError_t launch_unreachable(int32_t* count, const int32_t* seq_lens, const int32_t* query_lens,
                               int window, const int32_t* windows, int block_shift, int batch,
                               cudaStream_t stream);

// Staging copies for the host-buffer entry point: up to kMaxStageCopies
// buffers copied by one kernel (one launch instead of one DMA copy per
// buffer).  Sources are device addresses of pinned, mapped host buffers.
constexpr int kMaxStageCopies = 6;
struct StageCopy {
  const void* src;
  void* dst;
  unsigned long long units;  // number of `unit`-byte pieces
  int unit;                  // 16, 4 or 1: the widest both addresses and the size allow
  int first_block;           // the copy's CTAs are [first_block, next copy's first_block)
};
struct StageArgs {
  StageCopy c[kMaxStageCopies];
  int n;
  int blocks;  // grid size
};

// Launches the staging copies; the next kernel on the stream may be launched
// while they run (it waits for their completion before reading anything).
cudaError_t launch_stage(const StageArgs& s, cudaStream_t stream);

// Reads (and optionally clears) the device status word.
cudaError_t read_status(unsigned int* status, bool clear, cudaStream_t stream);

// Unique id of the calling thread's current CUDA context, or 0 when there is
// none yet (or the driver cannot say).  cudaDeviceReset replaces a device's
// primary context, and kernel attributes and symbol addresses belong to the
// context, so state cached across calls is keyed by this id.
unsigned long long context_id();

}  // namespace pa
