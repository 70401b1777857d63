// pa_kernels.cu -- sm_100a kernels of libpagedattn: the split-K partition
// kernel (CUDA-core FMA variant), the log-sum-exp reduce, and the
// visible-range kernel.  All device code lives in this one translation unit
// so the status word needs no relocatable device code.
//
// Method: ExecuTorch PR #18759 "SDPA decode perf improvements for
// qwen-3.5-35B-A3B" (split-K flash-decoding: the KV sequence is partitioned
// across CTAs, each partition keeps a running max and sum, a reduce merges the
// partials) applied to a paged KV cache as gllm PR #116 "feat(backend):
// sliding-window PagedAttention" defines it (block tables, per-token window
// start).  Design for B200: one copy warp streams K/V rows of each partition
// through a shared-memory ring with the TMA engine's bulk copies
// (cp.async.bulk + mbarrier transaction counts); compute warps read each
// staged K/V row once for every query row of the GQA group.
#include <climits>

#include <cuda.h>

#include "pa_device.cuh"
#include "pa_kernels.cuh"

namespace pa {

namespace {

constexpr int TS = kStageTokens;  // tokens per stage
constexpr int LPT = 8;            // lanes per token: each lane owns D/8 dims
constexpr int TPI = 32 / LPT;     // tokens per warp iteration
constexpr int ITERS = TS / TPI;   // warp iterations per stage
constexpr int CHUNK = 4;          // iterations per online-softmax update
constexpr unsigned FULL = 0xffffffffu;

template <int D>
struct FmaTraits {
  static constexpr int ROWB = D * 2;                // bytes per token row (bf16)
  static constexpr int CH = D / 64;                 // 16-byte chunks per lane per token
  static constexpr int NP = CH * 4;                 // float2 pairs per lane per row
  static constexpr int STAGE_BYTES = 2 * TS * ROWB; // K rows, then V rows
};

template <int D, int NCW>
struct CombineLayout {
  // per consumer warp, per token group (4), per row (4): partial acc and sum;
  // per consumer warp, per row: running max.
  static constexpr int ACC_FLOATS = NCW * 4 * 4 * D;
  static constexpr int L_FLOATS = NCW * 4 * 4;
  static constexpr int M_FLOATS = NCW * 4;
  static constexpr int BYTES = (ACC_FLOATS + L_FLOATS + M_FLOATS) * 4;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Partition kernel, CUDA-core FMA variant.
//
// CTA = (partition, kv head [x row slab], batch row).  Warp 0 copies; warps
// 1..NCW compute.  A compute warp owns a group of 4 query rows (q heads of the
// GQA group x query tokens) and a slice of each stage's tokens; 8 lanes share a
// token, each lane holding D/8 dims of q, K, V and the output accumulator.
// Scores are reduced across the 8 lanes with a transposing butterfly that
// leaves each lane one (row, token) score, so the softmax runs on 1 value per
// lane, then the 4 probabilities are broadcast back for the PV update.
// ---------------------------------------------------------------------------
template <int D, int NCW, int NSTAGE>
__global__ void __launch_bounds__(32 * (NCW + 1), 1)
    pa_partition_fma_kernel(const __grid_constant__ DecodeArgs a) {
  using T = FmaTraits<D>;
  using C = CombineLayout<D, NCW>;
  static_assert(C::BYTES <= NSTAGE * T::STAGE_BYTES, "combine area must fit in the ring");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTAGE * T::STAGE_BYTES);
  int* bt_s = reinterpret_cast<int*>(bars + 2 * NSTAGE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  const int kvh = blockIdx.y % a.num_kv_heads;
  const int slab = blockIdx.y / a.num_kv_heads;
  const int part = blockIdx.x;

  const int S = a.seq_lens[b];
  const int L = a.query_lens[b];
  const int w = a.windows ? a.windows[b] : a.window;
  if (L <= 0) return;
  const bool lead = (part == 0 && slab == 0 && kvh == 0 && threadIdx.x == 0);
  if (L > S || w < 0 || S > a.max_blocks_per_seq * a.block_size) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_BAD_ROW);
    return;
  }
  const int R = a.group * L;
  const int ulo = union_lo(S, L, w);
  const int A = ulo & ~(TS - 1);  // stages are aligned to 64-token boundaries
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (R > a.max_rows || nparts > a.max_parts) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_HINT);
    return;
  }
  const int row0 = slab * a.slab_rows;
  if (row0 >= R || part >= nparts) return;
  const int Rs = min(a.slab_rows, R - row0);
  const int p0 = A + part * a.part_tokens;
  const int p1 = min(S, p0 + a.part_tokens);
  const int nst = (p1 - p0 + TS - 1) / TS;
  const int jb0 = p0 >> a.block_shift;
  const int nbt = ((p1 - 1) >> a.block_shift) - jb0 + 1;

  // Block-table slice of this partition -> smem, checked against the pool.
  for (int i = threadIdx.x; i < nbt; i += blockDim.x) {
    int phys = a.block_tables[(size_t)b * a.max_blocks_per_seq + jb0 + i];
    if (phys < 0 || phys >= a.num_blocks) {
      atomicOr(&g_pa_status, PA_DEV_BAD_BLOCK);
      phys = -1;
    }
    bt_s[i] = phys;
  }
  // Zero the ring once: a row a stage does not copy then holds zeros or an
  // earlier stage's in-span data, never uninitialised bits, so a masked
  // token's zero probability never meets a NaN.
  {
    uint4* z = reinterpret_cast<uint4*>(smem);
    for (int i = threadIdx.x; i < NSTAGE * T::STAGE_BYTES / 16; i += blockDim.x)
      z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);             // full: producer arrival + tx bytes
      mbar_init(smem_u32(&bars[NSTAGE + s]), NCW);  // empty: one arrival per compute warp
    }
    fence_mbar_init();
  }
  const int qoff = row_token_offset(a.query_lens, b, lane);
  __syncthreads();

  float* comb_acc = reinterpret_cast<float*>(smem);
  float* comb_l = comb_acc + C::ACC_FLOATS;
  float* comb_m = comb_l + C::L_FLOATS;
  const int NRG = (Rs + 3) >> 2;  // row groups of 4 in this slab

  if (warp == 0) {
    // ------------------------------ copy warp ------------------------------
    bool ok = true;
    int issued = 0;
    for (int k = 0; k < nst; ++k) {
      const int s = k % NSTAGE;
      if (k >= NSTAGE) {
        bool got = true;
        if (lane == 0) got = mbar_wait(smem_u32(&bars[NSTAGE + s]), ((k / NSTAGE) - 1) & 1);
        ok = __shfl_sync(FULL, got, 0);
        if (!ok) break;
      }
      const int c0 = p0 + k * TS;
      const int ta = max(c0, ulo), te = min(c0 + TS, p1);
      const int jf = ta >> a.block_shift;
      const int npc = ((te - 1) >> a.block_shift) - jf + 1;  // block pieces (<= 4 for BS >= 16)
      uint32_t my_bytes = 0, dsto = 0;
      const __nv_bfloat16* src = nullptr;
      if (lane < 2 * npc) {
        const bool isv = lane >= npc;
        const int jj = jf + (isv ? lane - npc : lane);
        const int t_a = max(ta, jj << a.block_shift);
        const int t_e = min(te, (jj + 1) << a.block_shift);
        const int phys = bt_s[jj - jb0];
        if (phys >= 0) {
          my_bytes = (uint32_t)(t_e - t_a) * T::ROWB;
          const size_t off =
              (((size_t)phys * a.num_kv_heads + kvh) * a.block_size + (t_a - (jj << a.block_shift))) *
              (size_t)D;
          src = (isv ? a.v_cache : a.k_cache) + off;
          dsto = s * T::STAGE_BYTES + (isv ? TS * T::ROWB : 0) + (t_a - c0) * T::ROWB;
        }
      }
      const uint32_t total = __reduce_add_sync(FULL, my_bytes);
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&bars[s]), total);
      __syncwarp();
      if (my_bytes) bulk_g2s(smem_u32(smem) + dsto, src, my_bytes, smem_u32(&bars[s]));
      issued = k + 1;
    }
    // Drain: make sure no copy this warp issued is still in flight.
    if (lane == 0) {
      for (int k = max(0, issued - NSTAGE); k < issued; ++k)
        mbar_wait(smem_u32(&bars[k % NSTAGE]), (k / NSTAGE) & 1);
    }
    __syncwarp();
  } else {
    // ----------------------------- compute warps ---------------------------
    const int cw = warp - 1;
    const int rg = cw % NRG;
    const int slice = cw / NRG;
    const int nslice = (NCW - 1 - rg) / NRG + 1;
    const int tg = lane >> 3;   // token group: which of the iteration's 4 tokens
    const int l8 = lane & 7;    // lane within the token group
    const int rl = 2 * ((l8 >> 2) & 1) + ((l8 >> 1) & 1);  // row this lane scores

    int lo_r = INT_MAX, hi_r = INT_MIN;  // padding rows see nothing
    if (rg * 4 + rl < Rs) query_range(S, L, (row0 + rg * 4 + rl) / a.group, w, lo_r, hi_r);

    float2 qf[4][T::NP];
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
      const int rloc = rg * 4 + r4;
#pragma unroll
      for (int x = 0; x < T::NP; ++x) qf[r4][x] = make_float2(0.f, 0.f);
      if (rloc < Rs) {
        const int rr = row0 + rloc;
        const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
        const __nv_bfloat16* qp =
            a.q + ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + l8 * 8;
#pragma unroll
        for (int c = 0; c < T::CH; ++c) {
          const uint4 u = ldg128_nc(qp + c * 64);
          const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            const float2 f = bf2_to_f2(ws[pp]);
            qf[r4][c * 4 + pp] = make_float2(f.x * a.scale_log2, f.y * a.scale_log2);
          }
        }
      }
    }

    float2 acc[4][T::NP];
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4)
#pragma unroll
      for (int x = 0; x < T::NP; ++x) acc[r4][x] = make_float2(0.f, 0.f);
    float m_run = kNegInf, l_run = 0.f;

    for (int k = 0; k < nst; ++k) {
      const int s = k % NSTAGE;
      const bool got = mbar_wait(smem_u32(&bars[s]), (k / NSTAGE) & 1);
      if (!__all_sync(FULL, got)) break;
      const uint8_t* Ks = smem + s * T::STAGE_BYTES;
      const uint8_t* Vs = Ks + TS * T::ROWB;
      const int c0 = p0 + k * TS;

      for (int m0 = 0; slice + nslice * m0 < ITERS; m0 += CHUNK) {
        float sc[CHUNK];
#pragma unroll
        for (int u = 0; u < CHUNK; ++u) {
          const int it = slice + nslice * (m0 + u);
          sc[u] = kNegInf;
          if (it < ITERS) {
            const int tt = it * TPI + tg;
            float2 a4[4];
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4) a4[r4] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < T::CH; ++c) {
              const uint4 kk = lds128(Ks + tt * T::ROWB + c * 128 + l8 * 16);
              const uint32_t ws[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) {
                const float2 kf = bf2_to_f2(ws[pp]);
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) a4[r4] = __ffma2_rn(qf[r4][c * 4 + pp], kf, a4[r4]);
              }
            }
            const float s0 = a4[0].x + a4[0].y, s1 = a4[1].x + a4[1].y;
            const float s2 = a4[2].x + a4[2].y, s3 = a4[3].x + a4[3].y;
            // transposing butterfly over the 8 lanes of the token
            const bool b2 = (l8 & 4) != 0;
            float k0 = b2 ? s2 : s0, k1 = b2 ? s3 : s1;
            k0 += __shfl_xor_sync(FULL, b2 ? s0 : s2, 4);
            k1 += __shfl_xor_sync(FULL, b2 ? s1 : s3, 4);
            const bool b1 = (l8 & 2) != 0;
            float kv = b1 ? k1 : k0;
            kv += __shfl_xor_sync(FULL, b1 ? k0 : k1, 2);
            kv += __shfl_xor_sync(FULL, kv, 1);
            const int t = c0 + tt;
            sc[u] = (t >= lo_r && t < hi_r) ? kv : kNegInf;
          }
        }
        // online softmax over this chunk (log2 domain)
        float mc = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
        mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 8));
        mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 16));
        const float m_new = fmaxf(m_run, mc);
        const bool none = (m_new == kNegInf);
        const float m_use = none ? 0.f : m_new;
        const float alpha = none ? 1.f : ex2(m_run - m_use);
        float p[CHUNK];
        float psum = 0.f;
#pragma unroll
        for (int u = 0; u < CHUNK; ++u) {
          p[u] = ex2(sc[u] - m_use);
          psum += p[u];
        }
        l_run = l_run * alpha + psum;
        m_run = m_new;
        if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4) {
            const float ar = __shfl_sync(FULL, alpha, 2 * r4);
            const float2 a2 = make_float2(ar, ar);
#pragma unroll
            for (int x = 0; x < T::NP; ++x) acc[r4][x] = __fmul2_rn(acc[r4][x], a2);
          }
        }
#pragma unroll
        for (int u = 0; u < CHUNK; ++u) {
          const int it = slice + nslice * (m0 + u);
          if (it < ITERS) {
            const int tt = it * TPI + tg;
            float2 pr[4];
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4) {
              const float pv = __shfl_sync(FULL, p[u], (lane & 24) | (2 * r4));
              pr[r4] = make_float2(pv, pv);
            }
#pragma unroll
            for (int c = 0; c < T::CH; ++c) {
              const uint4 vv = lds128(Vs + tt * T::ROWB + c * 128 + l8 * 16);
              const uint32_t ws[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) {
                const float2 vf = bf2_to_f2(ws[pp]);
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4)
                  acc[r4][c * 4 + pp] = __ffma2_rn(pr[r4], vf, acc[r4][c * 4 + pp]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[NSTAGE + s]));
    }

    // All compute warps are done reading the ring; reuse it for the combine.
    named_bar_sync(1, NCW * 32);
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
      float* dstp = comb_acc + ((cw * 4 + tg) * 4 + r4) * D + l8 * 8;
#pragma unroll
      for (int c = 0; c < T::CH; ++c) {
        *reinterpret_cast<float4*>(dstp + c * 64) =
            make_float4(acc[r4][c * 4 + 0].x, acc[r4][c * 4 + 0].y, acc[r4][c * 4 + 1].x,
                        acc[r4][c * 4 + 1].y);
        *reinterpret_cast<float4*>(dstp + c * 64 + 4) =
            make_float4(acc[r4][c * 4 + 2].x, acc[r4][c * 4 + 2].y, acc[r4][c * 4 + 3].x,
                        acc[r4][c * 4 + 3].y);
      }
    }
    if ((l8 & 1) == 0) {
      comb_l[(cw * 4 + tg) * 4 + rl] = l_run;
      if (tg == 0) comb_m[cw * 4 + rl] = m_run;
    }
  }
  __syncthreads();

  // ----------------- merge the compute warps' partials --------------------
  for (int idx = threadIdx.x; idx < Rs * D; idx += blockDim.x) {
    const int rloc = idx / D;
    const int d = idx - rloc * D;
    const int rgi = rloc >> 2, r4 = rloc & 3;
    float M = kNegInf;
    for (int c = rgi; c < NCW; c += NRG) M = fmaxf(M, comb_m[c * 4 + r4]);
    float Z = 0.f, O = 0.f;
    if (M != kNegInf) {
      for (int c = rgi; c < NCW; c += NRG) {
        const float sc = ex2(comb_m[c * 4 + r4] - M);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          Z += sc * comb_l[(c * 4 + g) * 4 + r4];
          O += sc * comb_acc[((c * 4 + g) * 4 + r4) * D + d];
        }
      }
    }
    const int rr = row0 + rloc;
    if (nparts == 1) {
      const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
      a.dst[((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + d] =
          __float2bfloat16_rn(O / Z);
    } else {
      const size_t base =
          ((size_t)(b * a.num_kv_heads + kvh) * a.max_parts + part) * a.max_rows + rr;
      a.ws_o[base * D + d] = Z > 0.f ? O / Z : 0.f;
      if (d == 0) a.ws_lse[base] = Z > 0.f ? M + lg2(Z) : kNegInf;
    }
  }
}

// ---------------------------------------------------------------------------
// Partition kernel, tensor-core variant (rows = GQA group x query tokens form
// a dense tile: group x queryLen >= 8).
//
// Staging: the copy warp loads whole KV boxes (one block for 16/32/64-token
// blocks, a 64-token slice of larger blocks) with 2-D tiled TMA copies and
// the 128-byte swizzle, so each stage holds K then V as [D/64][64 tokens]
// [128 B] with 16-byte chunk c of token t stored at chunk c ^ (t & 7): every
// ldmatrix below reads 8 distinct bank groups.  Compute: each compute warp
// owns a 16-row M tile (rows past the real ones are padding) and a slice of
// the stage's 16-token chunks; S = Q K^T and O += P V run as m16n8k16 bf16
// MMAs with fp32 accumulation, P staying in registers between the two.
// Tokens a box brings in from outside the row's visible union (the head of
// the first block, the tail of the last) get score -inf and their V lanes
// are zeroed in registers, so uninitialised cache slots never reach O.
// ---------------------------------------------------------------------------
template <int D>
struct MmaTraits {
  static constexpr int HALVES = D / 64;
  static constexpr int HALF_BYTES = TS * 128;
  static constexpr int KV_BYTES = HALVES * HALF_BYTES;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;
  static constexpr int KSTEPS = D / 16;
  static constexpr int NT = D / 8;  // 8-wide output column tiles
};

template <int D, int NCW>
struct MmaCombine {
  static constexpr int ACC_FLOATS = NCW * 16 * D;
  static constexpr int L_FLOATS = NCW * 16;
  static constexpr int M_FLOATS = NCW * 16;
  static constexpr int BYTES = (ACC_FLOATS + L_FLOATS + M_FLOATS) * 4;
};

// Byte offset of 16-byte chunk `chunk` (0 .. D/8-1) of stage token row t.
__device__ __forceinline__ uint32_t swz(int t, int chunk) {
  return (uint32_t)((chunk >> 3) * (TS * 128) + t * 128 + (((chunk & 7) ^ (t & 7)) << 4));
}

template <int D, int NCW, int NSTAGE>
__global__ void __launch_bounds__(32 * (NCW + 1), 1)
    pa_partition_mma_kernel(const __grid_constant__ DecodeArgs a,
                            const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
  using T = MmaTraits<D>;
  using C = MmaCombine<D, NCW>;
  static_assert(C::BYTES <= NSTAGE * T::STAGE_BYTES, "combine area must fit in the ring");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  // 128-byte-swizzled TMA destinations must sit on 1024-byte boundaries.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTAGE * T::STAGE_BYTES);
  int* bt_s = reinterpret_cast<int*>(bars + 2 * NSTAGE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  const int kvh = blockIdx.y % a.num_kv_heads;
  const int slab = blockIdx.y / a.num_kv_heads;
  const int part = blockIdx.x;

  const int S = a.seq_lens[b];
  const int L = a.query_lens[b];
  const int w = a.windows ? a.windows[b] : a.window;
  if (L <= 0) return;
  const bool lead = (part == 0 && slab == 0 && kvh == 0 && threadIdx.x == 0);
  if (L > S || w < 0 || S > a.max_blocks_per_seq * a.block_size) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_BAD_ROW);
    return;
  }
  const int R = a.group * L;
  const int ulo = union_lo(S, L, w);
  const int A = ulo & ~(TS - 1);
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (R > a.max_rows || nparts > a.max_parts) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_HINT);
    return;
  }
  const int row0 = slab * a.slab_rows;
  if (row0 >= R || part >= nparts) return;
  const int Rs = min(a.slab_rows, R - row0);
  const int p0 = A + part * a.part_tokens;
  const int p1 = min(S, p0 + a.part_tokens);
  const int nst = (p1 - p0 + TS - 1) / TS;
  const int jb0 = p0 >> a.block_shift;
  const int nbt = ((p1 - 1) >> a.block_shift) - jb0 + 1;

  for (int i = threadIdx.x; i < nbt; i += blockDim.x) {
    int phys = a.block_tables[(size_t)b * a.max_blocks_per_seq + jb0 + i];
    if (phys < 0 || phys >= a.num_blocks) {
      atomicOr(&g_pa_status, PA_DEV_BAD_BLOCK);
      phys = -1;
    }
    bt_s[i] = phys;
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[NSTAGE + s]), NCW);
    }
    fence_mbar_init();
  }
  const int qoff = row_token_offset(a.query_lens, b, lane);
  __syncthreads();

  float* comb_acc = reinterpret_cast<float*>(smem);
  float* comb_l = comb_acc + C::ACC_FLOATS;
  float* comb_m = comb_l + C::L_FLOATS;
  const int NMT = (Rs + 15) >> 4;  // 16-row M tiles in this slab

  if (warp == 0) {
    // ------------------------------ copy warp ------------------------------
    const int BR = min(a.block_size, TS);  // rows per box
    const int nbox = TS / BR;
    const int nitem = nbox * 2 * T::HALVES;  // (box, K/V, half) per lane
    const uint32_t box_bytes = (uint32_t)BR * 128u;
    int issued = 0;
    for (int k = 0; k < nst; ++k) {
      const int s = k % NSTAGE;
      if (k >= NSTAGE) {
        bool got = true;
        if (lane == 0) got = mbar_wait(smem_u32(&bars[NSTAGE + s]), ((k / NSTAGE) - 1) & 1);
        if (!__shfl_sync(FULL, got, 0)) break;
      }
      const int c0 = p0 + k * TS;
      const int ta = max(c0, ulo), te = min(c0 + TS, p1);
      bool mine = false;
      uint32_t dst = 0;
      int x = 0, y = 0, isv = 0;
      if (lane < nitem) {
        const int j = lane / (2 * T::HALVES);
        const int rem = lane - j * (2 * T::HALVES);
        isv = rem / T::HALVES;
        const int h = rem - isv * T::HALVES;
        const int bt0 = c0 + j * BR;
        if (bt0 + BR > ta && bt0 < te) {
          const int jj = bt0 >> a.block_shift;
          const int phys = bt_s[jj - jb0];
          if (phys >= 0) {
            mine = true;
            x = h * 64;
            y = (phys * a.num_kv_heads + kvh) * a.block_size + (bt0 - (jj << a.block_shift));
            dst = s * T::STAGE_BYTES + isv * T::KV_BYTES + h * T::HALF_BYTES + j * BR * 128;
          }
        }
      }
      const uint32_t nload = __popc(__ballot_sync(FULL, mine));
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&bars[s]), nload * box_bytes);
      __syncwarp();
      if (mine)
        tma_load_2d(smem_u32(smem) + dst, isv ? static_cast<const void*>(&tmv)
                                              : static_cast<const void*>(&tmk),
                    x, y, smem_u32(&bars[s]));
      issued = k + 1;
    }
    if (lane == 0) {
      for (int k = max(0, issued - NSTAGE); k < issued; ++k)
        mbar_wait(smem_u32(&bars[k % NSTAGE]), (k / NSTAGE) & 1);
    }
    __syncwarp();
  } else {
    // ----------------------------- compute warps ---------------------------
    const int cw = warp - 1;
    const int mt = cw % NMT;
    const int slice = cw / NMT;
    const int nslice = (NCW - 1 - mt) / NMT + 1;
    const int quad = lane >> 2, qi = lane & 3;
    const int ra = mt * 16 + quad, rb = ra + 8;  // slab-local rows of this thread
    int lo_a = INT_MAX, hi_a = INT_MIN, lo_b = INT_MAX, hi_b = INT_MIN;
    if (ra < Rs) query_range(S, L, (row0 + ra) / a.group, w, lo_a, hi_a);
    if (rb < Rs) query_range(S, L, (row0 + rb) / a.group, w, lo_b, hi_b);
    int lo_max, hi_min, dummy;
    query_range(S, L, L - 1, w, lo_max, dummy);  // the last token sees the latest start
    query_range(S, L, 0, w, dummy, hi_min);      // the first token sees the earliest end

    // Q as A fragments (bf16, exact); the scale is applied to the fp32 scores.
    uint32_t qa[T::KSTEPS][4];
    {
      const uint32_t* qrow[2] = {nullptr, nullptr};
      const int rows[2] = {ra, rb};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (rows[e] < Rs) {
          const int rr = row0 + rows[e];
          const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
          qrow[e] = reinterpret_cast<const uint32_t*>(
              a.q + ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D);
        }
      }
#pragma unroll
      for (int ks = 0; ks < T::KSTEPS; ++ks) {
        const int col2 = ks * 8 + qi;  // bf16-pair index of column ks*16 + 2*qi
        qa[ks][0] = qrow[0] ? __ldg(qrow[0] + col2) : 0u;
        qa[ks][1] = qrow[1] ? __ldg(qrow[1] + col2) : 0u;
        qa[ks][2] = qrow[0] ? __ldg(qrow[0] + col2 + 4) : 0u;
        qa[ks][3] = qrow[1] ? __ldg(qrow[1] + col2 + 4) : 0u;
      }
    }

    float o[T::NT][4];
#pragma unroll
    for (int n = 0; n < T::NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_a = kNegInf, m_b = kNegInf, l_a = 0.f, l_b = 0.f;

    for (int k = 0; k < nst; ++k) {
      const int s = k % NSTAGE;
      const bool got = mbar_wait(smem_u32(&bars[s]), (k / NSTAGE) & 1);
      if (!__all_sync(FULL, got)) break;
      const uint32_t Ks = smem_u32(smem + s * T::STAGE_BYTES);
      const uint32_t Vs = Ks + T::KV_BYTES;
      const int c0 = p0 + k * TS;
      const bool all_valid = (c0 >= lo_max) && (c0 + TS <= hi_min);
      const bool boundary = (c0 < ulo) || (c0 + TS > p1);

      for (int ch = slice; ch < TS / 16; ch += nslice) {
        const int tb = ch * 16;
        float sc[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < T::KSTEPS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(Ks + swz(tb + ((lane >> 4) << 3) + (lane & 7), ks * 2 + ((lane >> 3) & 1)), b0,
                  b1, b2, b3);
          mma_bf16_16816(sc[0], qa[ks], b0, b1);
          mma_bf16_16816(sc[1], qa[ks], b2, b3);
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[n][e] *= a.scale_log2;
        if (!all_valid) {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t = c0 + tb + n * 8 + 2 * qi + (e & 1);
              const bool ok = (e < 2) ? (t >= lo_a && t < hi_a) : (t >= lo_b && t < hi_b);
              sc[n][e] = ok ? sc[n][e] : kNegInf;
            }
        }
        float mx_a = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        float mx_b = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(FULL, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(FULL, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(FULL, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(FULL, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float mu_a = (mn_a == kNegInf) ? 0.f : mn_a;
        const float mu_b = (mn_b == kNegInf) ? 0.f : mn_b;
        const float al_a = (mn_a == kNegInf) ? 1.f : ex2(m_a - mu_a);
        const float al_b = (mn_b == kNegInf) ? 1.f : ex2(m_b - mu_b);
        m_a = mn_a;
        m_b = mn_b;
        float p[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          p[n][0] = ex2(sc[n][0] - mu_a);
          p[n][1] = ex2(sc[n][1] - mu_a);
          p[n][2] = ex2(sc[n][2] - mu_b);
          p[n][3] = ex2(sc[n][3] - mu_b);
        }
        l_a = l_a * al_a + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
        l_b = l_b * al_b + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
        if (__any_sync(FULL, al_a != 1.f || al_b != 1.f)) {
#pragma unroll
          for (int n = 0; n < T::NT; ++n) {
            o[n][0] *= al_a;
            o[n][1] *= al_a;
            o[n][2] *= al_b;
            o[n][3] *= al_b;
          }
        }
        const uint32_t pa[4] = {pack_bf16x2(p[0][0], p[0][1]), pack_bf16x2(p[0][2], p[0][3]),
                                pack_bf16x2(p[1][0], p[1][1]), pack_bf16x2(p[1][2], p[1][3])};
        uint32_t mk_lo = 0xffffffffu, mk_hi = 0xffffffffu;
        if (boundary) {
          const int t = c0 + tb + 2 * qi;
          auto in = [&](int u) { return u >= ulo && u < p1; };
          mk_lo = (in(t) ? 0x0000ffffu : 0u) | (in(t + 1) ? 0xffff0000u : 0u);
          mk_hi = (in(t + 8) ? 0x0000ffffu : 0u) | (in(t + 9) ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int dp = 0; dp < T::NT / 2; ++dp) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_t(Vs + swz(tb + (((lane >> 3) & 1) << 3) + (lane & 7), dp * 2 + (lane >> 4)), v0,
                    v1, v2, v3);
          v0 &= mk_lo;
          v1 &= mk_hi;
          v2 &= mk_lo;
          v3 &= mk_hi;
          mma_bf16_16816(o[2 * dp], pa, v0, v1);
          mma_bf16_16816(o[2 * dp + 1], pa, v2, v3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[NSTAGE + s]));
    }

    named_bar_sync(1, NCW * 32);
#pragma unroll
    for (int n = 0; n < T::NT; ++n) {
      const int d = n * 8 + 2 * qi;
      *reinterpret_cast<float2*>(comb_acc + (cw * 16 + quad) * D + d) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(comb_acc + (cw * 16 + quad + 8) * D + d) =
          make_float2(o[n][2], o[n][3]);
    }
    l_a += __shfl_xor_sync(FULL, l_a, 1);
    l_a += __shfl_xor_sync(FULL, l_a, 2);
    l_b += __shfl_xor_sync(FULL, l_b, 1);
    l_b += __shfl_xor_sync(FULL, l_b, 2);
    if (qi == 0) {
      comb_l[cw * 16 + quad] = l_a;
      comb_l[cw * 16 + quad + 8] = l_b;
      comb_m[cw * 16 + quad] = m_a;
      comb_m[cw * 16 + quad + 8] = m_b;
    }
  }
  __syncthreads();

  // ----------------- merge the compute warps' partials --------------------
  for (int idx = threadIdx.x; idx < Rs * D; idx += blockDim.x) {
    const int rloc = idx / D;
    const int d = idx - rloc * D;
    const int mti = rloc >> 4, r16 = rloc & 15;
    float M = kNegInf;
    for (int c = mti; c < NCW; c += NMT) M = fmaxf(M, comb_m[c * 16 + r16]);
    float Z = 0.f, O = 0.f;
    if (M != kNegInf) {
      for (int c = mti; c < NCW; c += NMT) {
        const float sc = ex2(comb_m[c * 16 + r16] - M);
        Z += sc * comb_l[c * 16 + r16];
        O += sc * comb_acc[(c * 16 + r16) * D + d];
      }
    }
    const int rr = row0 + rloc;
    if (nparts == 1) {
      const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
      a.dst[((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + d] =
          __float2bfloat16_rn(O / Z);
    } else {
      const size_t base =
          ((size_t)(b * a.num_kv_heads + kvh) * a.max_parts + part) * a.max_rows + rr;
      a.ws_o[base * D + d] = Z > 0.f ? O / Z : 0.f;
      if (d == 0) a.ws_lse[base] = Z > 0.f ? M + lg2(Z) : kNegInf;
    }
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp reduce (ExecuTorch PR #18759, the split-K reduce kernel):
// per (row, kv head, batch row): M = max_p lse_p, w_p = 2^(lse_p - M),
// dst = sum_p w_p O_p / sum_p w_p.  Partials are normalised, so the weights
// carry each partition's softmax mass.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pa_reduce_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int NT = 256;
  constexpr int DQ = D / 4;
  constexpr int NPG = NT / DQ;
  __shared__ float red[NT / 32];
  __shared__ float4 pacc[NT];
  __shared__ float s_bcast;
  __shared__ int s_qoff;

  const int rr = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int S = a.seq_lens[b];
  const int L = a.query_lens[b];
  const int w = a.windows ? a.windows[b] : a.window;
  if (L <= 0 || L > S || w < 0 || S > a.max_blocks_per_seq * a.block_size) return;
  const int R = a.group * L;
  if (rr >= R || R > a.max_rows) return;
  const int A = union_lo(S, L, w) & ~(kStageTokens - 1);
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (nparts <= 1 || nparts > a.max_parts) return;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp == 0) {
    const int q0 = row_token_offset(a.query_lens, b, lane);
    if (lane == 0) s_qoff = q0;
  }
  const size_t ubase = (size_t)(b * a.num_kv_heads + kvh) * a.max_parts;
  const float* lse = a.ws_lse + ubase * a.max_rows + rr;

  float m = kNegInf;
  for (int p = tid; p < nparts; p += NT) m = fmaxf(m, lse[(size_t)p * a.max_rows]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (tid == 0) {
    float x = red[0];
    for (int i = 1; i < NT / 32; ++i) x = fmaxf(x, red[i]);
    s_bcast = x;
  }
  __syncthreads();
  const float M = s_bcast;
  __syncthreads();

  float z = 0.f;
  for (int p = tid; p < nparts; p += NT) z += ex2(lse[(size_t)p * a.max_rows] - M);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
  if (lane == 0) red[warp] = z;

  const int dq = tid % DQ, pg = tid / DQ;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p = pg; p < nparts; p += NPG) {
    const float wt = ex2(lse[(size_t)p * a.max_rows] - M);
    const float4 o =
        *reinterpret_cast<const float4*>(a.ws_o + ((ubase + p) * a.max_rows + rr) * D + dq * 4);
    acc.x += wt * o.x;
    acc.y += wt * o.y;
    acc.z += wt * o.z;
    acc.w += wt * o.w;
  }
  pacc[tid] = acc;
  __syncthreads();
  if (pg == 0) {
    float Z = 0.f;
    for (int i = 0; i < NT / 32; ++i) Z += red[i];
    for (int g = 1; g < NPG; ++g) {
      const float4 o = pacc[g * DQ + dq];
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }
    const float inv = 1.f / Z;
    const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
    __nv_bfloat16* dp =
        a.dst + ((size_t)(s_qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + dq * 4;
    const __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&lo2);
    packed.y = *reinterpret_cast<const uint32_t*>(&hi2);
    *reinterpret_cast<uint2*>(dp) = packed;
  }
}

// ---------------------------------------------------------------------------
// Visible ranges of every query token (one CTA; block-wide scan of queryLens
// gives each row's packed offset).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) pa_ranges_kernel(int32_t* lo, int32_t* hi,
                                                          const int32_t* seq_lens,
                                                          const int32_t* query_lens, int window,
                                                          const int32_t* windows, int batch) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < batch; base += blockDim.x) {
    const int b = base + tid;
    int L = 0, S = 0, w = window;
    if (b < batch) {
      L = query_lens[b];
      S = seq_lens[b];
      if (windows) w = windows[b];
      if (L < 0 || L > S || w < 0) {
        atomicOr(&g_pa_status, PA_DEV_BAD_ROW);
        L = L < 0 ? 0 : L;
      }
    }
    int x = L;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int v = lane < nwarps ? wsum[lane] : 0;
      const int incl = v;
      int e = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, e, o);
        if (lane >= o) e += y;
      }
      wsum[lane] = e - incl;  // exclusive prefix of warp totals
    }
    __syncthreads();
    const int off = carry + wsum[warp] + x - L;
    if (b < batch) {
      for (int i = 0; i < L; ++i) {
        int l, h;
        query_range(S, L, i, w, l, h);
        lo[off + i] = l;
        hi[off + i] = h;
      }
    }
    __syncthreads();
    if (tid == blockDim.x - 1) carry = off + L;
    __syncthreads();
  }
}

template <int D, int NCW, int NSTAGE>
cudaError_t launch_fma_t(const DecodeArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = pa_partition_fma_kernel<D, NCW, NSTAGE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 32 * (NCW + 1), smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int NCW, int NSTAGE>
int occupancy_fma_t(size_t smem) {
  auto kern = pa_partition_fma_kernel<D, NCW, NSTAGE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * (NCW + 1), smem) != cudaSuccess)
    return 0;
  return n;
}

template <int D, int NCW, int NSTAGE>
cudaError_t launch_mma_t(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                         dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = pa_partition_mma_kernel<D, NCW, NSTAGE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 32 * (NCW + 1), smem, stream>>>(a, tk, tv);
  return cudaGetLastError();
}

template <int D, int NCW, int NSTAGE>
int occupancy_mma_t(size_t smem) {
  auto kern = pa_partition_mma_kernel<D, NCW, NSTAGE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * (NCW + 1), smem) != cudaSuccess)
    return 0;
  return n;
}

}  // namespace

size_t mma_smem_bytes(int head_dim, int stages, int part_tokens, int block_size) {
  const size_t ring = (size_t)stages * 2 * TS * head_dim * 2;
  const size_t nbt = (size_t)part_tokens / block_size + 2;
  return 1024 + ring + 2 * (size_t)stages * sizeof(uint64_t) + nbt * sizeof(int);
}

#define PA_MMA_DISPATCH(CALL)                                                       \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 3) CALL(128, 4, 3); \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 4) CALL(64, 4, 4);

cudaError_t launch_partition_mma(const DecodeArgs& a, const KernelShape& k, const CUtensorMap& tk,
                                 const CUtensorMap& tv, dim3 grid, size_t smem,
                                 cudaStream_t stream) {
#define PA_CALL(D, N, S) return launch_mma_t<D, N, S>(a, tk, tv, grid, smem, stream)
  PA_MMA_DISPATCH(PA_CALL)
#undef PA_CALL
  return cudaErrorInvalidValue;
}

int occupancy_partition_mma(const KernelShape& k, size_t smem) {
#define PA_CALL(D, N, S) return occupancy_mma_t<D, N, S>(smem)
  PA_MMA_DISPATCH(PA_CALL)
#undef PA_CALL
  return 0;
}

size_t fma_smem_bytes(int head_dim, int stages, int part_tokens, int block_size) {
  const size_t ring = (size_t)stages * 2 * TS * head_dim * 2;
  const size_t nbt = (size_t)part_tokens / block_size + 2;
  return ring + 2 * (size_t)stages * sizeof(uint64_t) + nbt * sizeof(int);
}

#define PA_FMA_DISPATCH(CALL)                                           \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 3) CALL(128, 4, 3); \
  if (k.head_dim == 128 && k.consumer_warps == 8 && k.stages == 3) CALL(128, 8, 3); \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 4) CALL(64, 4, 4);   \
  if (k.head_dim == 64 && k.consumer_warps == 8 && k.stages == 4) CALL(64, 8, 4);

cudaError_t launch_partition_fma(const DecodeArgs& a, const KernelShape& k, dim3 grid,
                                 size_t smem, cudaStream_t stream) {
#define PA_CALL(D, N, S) return launch_fma_t<D, N, S>(a, grid, smem, stream)
  PA_FMA_DISPATCH(PA_CALL)
#undef PA_CALL
  return cudaErrorInvalidValue;
}

int occupancy_partition_fma(const KernelShape& k, size_t smem) {
#define PA_CALL(D, N, S) return occupancy_fma_t<D, N, S>(smem)
  PA_FMA_DISPATCH(PA_CALL)
#undef PA_CALL
  return 0;
}

cudaError_t launch_reduce(const DecodeArgs& a, cudaStream_t stream) {
  const dim3 grid(a.max_rows, a.num_kv_heads, a.batch);
  if (a.head_dim == 128)
    pa_reduce_kernel<128><<<grid, 256, 0, stream>>>(a);
  else if (a.head_dim == 64)
    pa_reduce_kernel<64><<<grid, 256, 0, stream>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_ranges(int32_t* lo, int32_t* hi, const int32_t* seq_lens,
                          const int32_t* query_lens, int window, const int32_t* windows,
                          int batch, cudaStream_t stream) {
  pa_ranges_kernel<<<1, 1024, 0, stream>>>(lo, hi, seq_lens, query_lens, window, windows, batch);
  return cudaGetLastError();
}

cudaError_t read_status(unsigned int* status, bool clear, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(status, g_pa_status, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  if (clear) {
    static const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_pa_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaStreamSynchronize(stream);
}

}  // namespace pa
