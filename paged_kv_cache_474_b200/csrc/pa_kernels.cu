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
#include <algorithm>
#include <climits>
#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include <cuda.h>
#include <cudaTypedefs.h>

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
__global__ void __launch_bounds__(32 * (NCW + 1), (NCW <= 4 ? 2 : 1))
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
  // Let the reduce grid launch now; it waits for this grid's completion
  // before reading any partial.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  float* comb_acc = reinterpret_cast<float*>(smem);
  float* comb_l = comb_acc + C::ACC_FLOATS;
  float* comb_m = comb_l + C::L_FLOATS;
  const int NRG = (Rs + 3) >> 2;  // row groups of 4 in this slab

  if (warp == 0) {
    // ------------------------------ copy warp ------------------------------
    const uint64_t kv_policy = l2_evict_first_policy();  // K/V rows are read once
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
          src = static_cast<const __nv_bfloat16*>(isv ? a.v_cache : a.k_cache) + off;
          dsto = s * T::STAGE_BYTES + (isv ? TS * T::ROWB : 0) + (t_a - c0) * T::ROWB;
        }
      }
      const uint32_t total = __reduce_add_sync(FULL, my_bytes);
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&bars[s]), total);
      __syncwarp();
      if (my_bytes)
        bulk_g2s_hint(smem_u32(smem) + dsto, src, my_bytes, smem_u32(&bars[s]), kv_policy);
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
// Partition kernel, tensor-core variant.
//
// Staging: the copy warp loads whole KV boxes (one block for 16/32/64-token
// blocks, a 64-token slice of larger blocks) with one 3-D tiled TMA copy per
// box and K/V, with the 128-byte swizzle.  A box lands as [D/64 halves]
// [BR rows][128 B] with 16-byte chunk c of row r stored at chunk c ^ (r & 7),
// so every ldmatrix below reads 8 distinct bank groups; a stage holds the K
// boxes, then the V boxes, of 64 tokens.
//
// Compute, with the KV tokens as the MMA's M dimension and the unit's query
// rows as N (8 rows per n-tile, so an 8-row GQA group is one dense tile):
//   S^T[16 tok x 8 rows] += K[16 tok x 16 d] . Q^T[16 d x 8 rows]
//   O^T[16 d x 8 rows]   += V^T[16 d x 16 tok] . P^T[16 tok x 8 rows]
// K and V^T come from smem by ldmatrix (V transposed on the fly), Q^T sits in
// registers for the whole partition, and P^T moves from the S^T accumulator
// layout to the B-operand layout with one movmatrix per 8x8 block.  Each
// thread's O^T columns are exactly the rows whose softmax statistics it
// holds, so the online-softmax rescale needs no data movement.  Tokens a box
// brings in from outside the row's visible union get score -inf and their V
// lanes are zeroed in registers, so uninitialised cache slots never reach O.
//
// FP8 e4m3 caches (F8): a token row is D bytes, staged the same way, and the
// MMAs run on f16 operands (e4m3 -> f16 is exact, one cvt per code pair; Q is
// converted to f16 once, P is packed as f16).  The reduction order over d and
// the order of O^T's rows are free, so the fragments are chosen to suit
// byte-wide data: a k-step takes one 16-byte chunk (16 dims); the thread
// that ldmatrix gives bytes 4c..4c+3 of a token row uses them as MMA k
// indices 2c, 2c+1, 2c+8, 2c+9, and Q^T is loaded with the same map.  For
// V^T, ldmatrix.trans over b16 pairs gives a thread two dims (2g, 2g+1) of
// two tokens; one byte permute regroups them by dim, so O^T row g of the
// tile is dim 2g and row g+8 is dim 2g+1.  q_scale * k_scale is folded into
// the score scale and v_scale into the output normalisation.
// ---------------------------------------------------------------------------
// Lazy running maximum of the tensor-core kernel's online softmax (log2
// units): 2^8 = 256 bounds the unnormalised probabilities, far inside the
// range of the bf16 and f16 P operands.
constexpr float kLazyMax = 8.f;

template <int D, bool F8>
struct MmaTraits {
  static constexpr int ROW_BYTES = F8 ? D : 2 * D;                  // one token of one kv head
  static constexpr int BOXW = ROW_BYTES < 128 ? ROW_BYTES : 128;    // swizzle span of a box row
  static constexpr int KV_BYTES = TS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;
  static constexpr int KSTEPS = D / 16;  // 16-wide reduction steps over d
  static constexpr int MD = D / 16;      // 16-dim M tiles of O^T
};

template <int D, int NCW, int N8>
struct MmaCombine {
  static constexpr int RT = 8 * N8;  // rows per warp tile
  static constexpr int LD = D + 4;   // padded row stride: conflict-free fragment stores
  static constexpr int ACC_FLOATS = NCW * RT * LD;
  static constexpr int L_FLOATS = NCW * RT;
  static constexpr int M_FLOATS = NCW * RT;
  static constexpr int BYTES = (ACC_FLOATS + L_FLOATS + M_FLOATS) * 4;
};

// Byte offset, within a box, of 16-byte chunk c = 2k + ck (ck in {0, 1}) of
// row lt (lt < 16, relative to a 16-row aligned chunk start).  128-byte box
// rows: half (c / 8) of the box (each half BR * 128 bytes), row lt, chunk
// position (c & 7) ^ (lt & 7) (the 128-byte swizzle); 64-byte rows (FP8,
// head_dim 64; 64-byte swizzle): chunk position (c & 3) ^ ((lt >> 1) & 3).
// 2k only touches chunk bits 1..3 and ck only bit 0, so the offset splits into
// a per-lane part, box_lane_off(lt, ck), computed once per warp, and a
// per-step part that is one XOR with a constant (and, for the second half,
// one add) once k is unrolled: (k >> 2) * half + (lane ^ (((2k) & 7) << 4)),
// or lane ^ (((2k) & 3) << 4) for 64-byte rows.
template <int BOXW>
__device__ __forceinline__ uint32_t box_lane_off(int lt, int ck) {
  if constexpr (BOXW == 128)
    return (uint32_t)(lt * 128 + ((ck ^ (lt & 7)) << 4));
  else
    return (uint32_t)(lt * 64 + ((ck ^ ((lt >> 1) & 3)) << 4));
}

template <int BOXW>
__device__ __forceinline__ uint32_t box_step_off(int k, uint32_t lane_off, uint32_t half) {
  if constexpr (BOXW == 128)
    return (uint32_t)(k >> 2) * half + (lane_off ^ (uint32_t)(((2 * k) & 7) << 4));
  else
    return lane_off ^ (uint32_t)(((2 * k) & 3) << 4);
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

struct LseAcc {
  float m, z;
  float4 o;
};

// (m, z, o) += (m2, z2, o2) with the larger maximum kept; -inf maxima weigh 0.
__device__ __forceinline__ void lse_merge(LseAcc& x, float m2, float z2, float4 o2) {
  const float mn = fmaxf(x.m, m2);
  const float f1 = mn == kNegInf ? 0.f : ex2(x.m - mn);
  const float f2 = mn == kNegInf ? 0.f : ex2(m2 - mn);
  x.z = x.z * f1 + z2 * f2;
  x.o.x = x.o.x * f1 + o2.x * f2;
  x.o.y = x.o.y * f1 + o2.y * f2;
  x.o.z = x.o.z * f1 + o2.z * f2;
  x.o.w = x.o.w * f1 + o2.w * f2;
  x.m = mn;
}

// ---------------------------------------------------------------------------
// Work-list merge (the reduce below, done by the unit's own CTAs).  Used by
// the work-list schedule, whose one-wave grid is launched cooperatively, so
// every CTA of a unit is resident: each CTA publishes its partial (fence, then
// an epoch-tagged arrival), waits until all nparts partials of its unit have
// arrived, then merges a share of the unit's outputs with a running
// log-sum-exp: up to 32 partials, one warp per row with its lanes over the
// dims; more, one CTA per (row, 16 dims) with its lanes over the partials in
// 64-byte slices.  Partials are read through L2 (ld.cg): other SMs wrote
// them during this kernel.
// ---------------------------------------------------------------------------
template <int D>
__device__ __noinline__ void merge_unit_partials(const DecodeArgs& a, int b, int kvh, int part,
                                                 int nparts, int row0, int Rs, int qoff,
                                                 int touched) {
  __shared__ int s_go;
  __shared__ float s_m[16], s_z[16];
  __shared__ float4 s_o[16][4];
  constexpr int C4 = D / 4;
  constexpr int DC = 16;         // many partials: dims per (row, slice) item
  constexpr int NSL = D / DC;    // slices per row
  constexpr int LPP = DC / 4;    // lanes per partial's slice (one float4 each)
  constexpr int PPW = 32 / LPP;  // partials per warp load
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const bool few = nparts <= 32;
  // Only CTAs with a share of the merge wait for the unit's arrivals; the
  // rest publish their partial and leave (fewer pollers on the counter).
  const bool share = few ? part * nw < Rs : part < Rs * NSL;
  __threadfence();
  __syncthreads();
  unsigned long long* cnt = a.done + (size_t)blockIdx.z * gridDim.y + blockIdx.y;
  if (threadIdx.x == 0) {
    if (!touched) epoch_touch(cnt, a.epoch);
    atomicAdd(cnt, 1ull);
    s_go = share && epoch_wait(cnt, a.epoch, (unsigned)nparts + a.wait_extra, a.wait_cycles);
    __threadfence();
  }
  __syncthreads();
  if (!s_go) return;
  const size_t ubase = (size_t)(b * a.num_kv_heads + kvh) * a.max_parts;
  auto store = [&](int rr, int c4, const LseAcc& acc) {
    const float inv = acc.z > 0.f ? 1.f / acc.z : 0.f;
    const int i = rr / a.group, jj = rr - (rr / a.group) * a.group;
    __nv_bfloat16* dp =
        a.dst + ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + jj) * D + c4 * 4;
    *reinterpret_cast<uint2*>(dp) = make_uint2(pack_bf16x2(acc.o.x * inv, acc.o.y * inv),
                                               pack_bf16x2(acc.o.z * inv, acc.o.w * inv));
  };
  if (few) {
    // Few partials: a warp per row, lanes over its dims (4 each), every
    // partial's loads issued before the first merge.
    constexpr int PB = 8;
    for (int r = part * nw + warp; r < Rs; r += nparts * nw) {
      const int rr = row0 + r;
      for (int c4 = lane; c4 < C4; c4 += 32) {
        LseAcc acc{kNegInf, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
        for (int p0 = 0; p0 < nparts; p0 += PB) {
          float l[PB];
          float4 o[PB];
#pragma unroll
          for (int u = 0; u < PB; ++u) {
            const size_t base = (ubase + p0 + u) * a.max_rows + rr;
            const bool in = p0 + u < nparts;
            l[u] = in ? __ldcg(a.ws_lse + base) : kNegInf;
            o[u] = in ? __ldcg(reinterpret_cast<const float4*>(a.ws_o + base * D) + c4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < PB; ++u) lse_merge(acc, l[u], 1.f, o[u]);
        }
        store(rr, c4, acc);
      }
    }
    return;
  }
  // Many partials: a CTA per (row, 16-dim slice).  Its warps split the
  // partials, LPP lanes reading one partial's slice (64 contiguous bytes), so
  // a warp load covers PPW partials; lanes, then warps (through shared
  // memory), merge with the same rescale.
  const int sub = lane / LPP, c4 = lane - (lane / LPP) * LPP;
  const size_t pst4 = (size_t)a.max_rows * D / 4;  // float4 stride between partials
  const int step = nw * PPW;
  constexpr int BATCH = 8;
  for (int it = part; it < Rs * NSL; it += nparts) {
    const int r = it / NSL, sl = it - (it / NSL) * NSL;
    const int rr = row0 + r;
    const float* lse = a.ws_lse + ubase * a.max_rows + rr;
    const float4* ob =
        reinterpret_cast<const float4*>(a.ws_o + (ubase * a.max_rows + rr) * D + sl * DC) + c4;
    LseAcc acc{kNegInf, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int p0 = warp * PPW + sub; p0 < nparts; p0 += BATCH * step) {
      float l[BATCH];
      float4 o[BATCH];
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const int p = p0 + u * step;
        l[u] = p < nparts ? __ldcg(lse + (size_t)p * a.max_rows) : kNegInf;
        o[u] = p < nparts ? __ldcg(ob + (size_t)p * pst4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < BATCH; ++u) lse_merge(acc, l[u], 1.f, o[u]);
    }
#pragma unroll
    for (int off = LPP; off < 32; off <<= 1) {
      const float m2 = __shfl_xor_sync(FULL, acc.m, off);
      const float z2 = __shfl_xor_sync(FULL, acc.z, off);
      float4 o2;
      o2.x = __shfl_xor_sync(FULL, acc.o.x, off);
      o2.y = __shfl_xor_sync(FULL, acc.o.y, off);
      o2.z = __shfl_xor_sync(FULL, acc.o.z, off);
      o2.w = __shfl_xor_sync(FULL, acc.o.w, off);
      lse_merge(acc, m2, z2, o2);
    }
    if (sub == 0) {
      s_o[warp][c4] = acc.o;
      if (c4 == 0) {
        s_m[warp] = acc.m;
        s_z[warp] = acc.z;
      }
    }
    __syncthreads();
    if (warp == 0 && lane < LPP) {
      LseAcc t{kNegInf, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
      for (int i = 0; i < nw; ++i) lse_merge(t, s_m[i], s_z[i], s_o[i][lane]);
      store(rr, sl * LPP + lane, t);
    }
    __syncthreads();
  }
}

// Register caps keep 4 (one n-tile) or 3 (two n-tiles) warps per SM
// sub-partition, so two CTAs fit per SM; head_dim 256 runs one CTA per SM
// (its 192 KB ring) and takes the larger cap for its wider accumulators.
template <int D, int NCW, int NSTAGE, int N8, bool F8, bool WL>
__global__ void __maxnreg__((N8 == 1 && D <= 128) ? 128 : 168)
    pa_partition_mma_kernel(const __grid_constant__ DecodeArgs a,
                            const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
  using T = MmaTraits<D, F8>;
  using C = MmaCombine<D, NCW, N8>;
  constexpr int RT = C::RT;
  // paired chunk processing (see the compute loop): FP8 caches, one n-tile,
  // an even ring depth, four compute warps, the static schedule
  constexpr bool PAIRABLE = F8 && N8 == 1 && NSTAGE % 2 == 0 && NCW == 4 && !WL;
  // ... whose compute warps refill their own halves (rings of at most four
  // stages: the six-stage ring serves one-wave grids, whose partitions need
  // about one refill per CTA, so there the extra code only costs registers)
  constexpr bool SELFREF = PAIRABLE && NSTAGE <= 4;
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
  // Paired mode (see the compute loop): a compute warp owns one half (32
  // tokens) of every other stage; with self-refill it also refills that half.
  const bool paired = PAIRABLE && a.pair_chunks;
  const bool selfref = SELFREF && a.pair_chunks;
  const int BR = a.box_rows;  // token rows per TMA box (<= 32 with self-refill)

  __shared__ int s_qoff;
  __shared__ float s_fac[NCW][64], s_rowm[64], s_rowz[64];  // warp-merge factors (rows <= 64)
  __shared__ int s_c0[WL ? NSTAGE : 1];  // work list: each slot's first token; -1: stop
  __shared__ int s_dtouch;                // work list: the arrival counter is this call's

  // Nothing here depends on the inputs: set up the pipeline while the
  // previous kernel on the stream may still be finishing (this kernel is
  // launched with programmatic stream serialization), then wait for it.
  if (threadIdx.x == 0) {
    if constexpr (WL) s_dtouch = 0;
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    // full: one arrival with the tx bytes per copy; empty: one arrival per
    // compute warp that consumes the stage (paired mode: two).  Self-refill
    // has no empty barriers: bars[NSTAGE + s] is the full barrier of slot s's
    // second half.
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[NSTAGE + s]), selfref ? 1u : paired ? 2u : (uint32_t)NCW);
    }
    fence_mbar_init();
  }
  // Every thread sees the initialised barriers before any of them can use
  // one.  With the early first stage (spec_first_stage) no warp waits for
  // another after this point before the main loops, so the copy warp's wait
  // for its table entries never holds up the compute warps' prologue.
  __syncthreads();
  if (warp == 1 && a.prefetch_stages > 0) {
    // L2 prefetch of the partition's first stages before the grid-dependency
    // wait, by a compute warp (they only wait for staged data after it; the
    // copy warp's path to its first copy stays as short as without it).  In a one-wave grid of window-free rows a partition starts at
    // part * part_tokens whatever the lengths, so only its block-table
    // entries are needed; the previous kernel may still rewrite them, so they
    // are read with relaxed loads and steer nothing but these prefetches
    // (clamped into the pool: every box lies inside the tensor map).  The
    // copies proper re-read the table after the wait and find the boxes in
    // L2 when nothing changed.
    const int c0 = part * a.part_tokens + a.prefetch_first * TS;
    const int br = BR;
    const int ntok = min(min(a.prefetch_stages * TS, a.part_tokens - a.prefetch_first * TS),
                         a.max_blocks_per_seq * a.block_size - c0);
    const int nitem = 2 * (max(ntok, 0) / br);
    const int32_t* tb = a.block_tables + (size_t)b * a.max_blocks_per_seq;
    for (int i = lane; i < nitem; i += 32) {
      const int t = c0 + (i >> 1) * br;
      const int jj = t >> a.block_shift;
      const int phys = min(max(ld_relaxed_s32(tb + jj), 0), a.num_blocks - 1);
      tma_prefetch_3d((i & 1) ? static_cast<const void*>(&tmv) : static_cast<const void*>(&tmk), 0,
                      (phys * a.num_kv_heads + kvh) * a.block_size + (t - (jj << a.block_shift)),
                      0);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int S = a.seq_lens[b];
  const int L = a.query_lens[b];
  const int w = a.windows ? a.windows[b] : a.window;
  // A row without a window starts its partitions at token 0, so the copy warp
  // can fetch the partition's block-table slice while the lengths are still
  // in flight (entries past the row's last block are read but never used).
  const bool spec_table = (!WL && a.windows == nullptr && a.window == 0);
  bool spec0 = false;  // copy warp: the partition's first stage is already in flight
  if (warp == 0 && spec_table) {
    const int sj0 = (part * a.part_tokens) >> a.block_shift;
    const int sn = min(a.part_tokens / a.block_size + 2, a.max_blocks_per_seq - sj0);
    for (int i = lane; i < sn; i += 32)
      bt_s[i] = a.block_tables[(size_t)b * a.max_blocks_per_seq + sj0 + i];
    // The first stage of a window-free partition starts at part * part_tokens
    // whatever the lengths say, so its boxes go out now, before the lengths
    // arrive.  Tokens past the row's end are masked like any stage's; table
    // entries outside the pool are clamped into it, so every copy stays inside
    // the tensor map (such an entry is still flagged below).
    const int c0 = part * a.part_tokens;
    if (a.spec_first_stage && c0 + TS <= a.max_blocks_per_seq * a.block_size) {
      __syncwarp();
      const int nitem0 = (TS / BR) * 2;
      const uint32_t bb = (uint32_t)BR * T::ROW_BYTES;
      uint32_t dst = 0, bar = smem_u32(&bars[0]);
      int y = 0, isv = 0;
      if (lane < nitem0) {
        const int jb = lane >> 1;
        isv = lane & 1;
        const int bt0 = c0 + jb * BR;
        const int jj = bt0 >> a.block_shift;
        const int phys = min(max(bt_s[jj - sj0], 0), a.num_blocks - 1);
        y = (phys * a.num_kv_heads + kvh) * a.block_size + (bt0 - (jj << a.block_shift));
        dst = isv * T::KV_BYTES + jb * bb;
        if (selfref && jb * BR >= TS / 2) bar = smem_u32(&bars[NSTAGE]);
      }
      if (lane == 0) {
        if (selfref) {  // each half: its own barrier, half the items
          mbar_arrive_expect_tx(smem_u32(&bars[0]), (uint32_t)(nitem0 / 2) * bb);
          mbar_arrive_expect_tx(smem_u32(&bars[NSTAGE]), (uint32_t)(nitem0 / 2) * bb);
        } else {
          mbar_arrive_expect_tx(smem_u32(&bars[0]), (uint32_t)nitem0 * bb);
        }
      }
      __syncwarp();
      if (lane < nitem0)
        tma_load_3d_hint(smem_u32(smem) + dst,
                         isv ? static_cast<const void*>(&tmv) : static_cast<const void*>(&tmk), 0,
                         y, 0, bar, l2_evict_first_policy());
      spec0 = true;
    }
  }
  // A CTA that leaves with a speculative stage in flight first waits for it.
  auto leave = [&]() {
    if (spec0 && lane == 0) {
      mbar_wait(smem_u32(&bars[0]), 0);
      if (selfref) mbar_wait(smem_u32(&bars[NSTAGE]), 0);
    }
  };
  if (L <= 0) {
    leave();
    return;
  }
  const bool lead = (part == 0 && slab == 0 && kvh == 0 && threadIdx.x == 0);
  if (L > S || w < 0 || S > a.max_blocks_per_seq * a.block_size) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_BAD_ROW);
    leave();
    return;
  }
  const int R = a.group * L;
  const int ulo = union_lo(S, L, w);
  const int A = ulo & ~(TS - 1);
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (R > a.max_rows || nparts > a.max_parts) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_HINT);
    leave();
    return;
  }
  const int row0 = slab * a.slab_rows;
  if (row0 >= R || part >= nparts) {
    leave();
    return;
  }
  const int Rs = min(a.slab_rows, R - row0);
  // Static schedule: this CTA's partition [p0, p1).  Work list: any stage of
  // the unit's span [A, S), so tokens are masked only at the span's ends.
  const int p0 = A + part * a.part_tokens;
  const int p1 = WL ? S : min(S, p0 + a.part_tokens);
  const int nst = (p1 - p0 + TS - 1) / TS;
  const int jb0 = p0 >> a.block_shift;
  const int nbt = ((p1 - 1) >> a.block_shift) - jb0 + 1;

  // Without the early first stage the warps meet once more here (measured a
  // little faster on the multi-wave and windowed workloads).
  if (!a.spec_first_stage) __syncthreads();
  // Let the reduce grid launch now; it waits for this grid's completion
  // before reading any partial.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  float* comb_acc = reinterpret_cast<float*>(smem);
  float* comb_l = comb_acc + C::ACC_FLOATS;
  float* comb_m = comb_l + C::L_FLOATS;
  const int NRT = (Rs + RT - 1) / RT;  // row tiles in this slab

  // A box is BR token rows of one (block, kv head): [halves][BR rows][BOXW bytes].
  const uint32_t box_bytes = (uint32_t)BR * T::ROW_BYTES;
  int qoff = 0;

  if (warp == 0) {
    // ------------------------------ copy warp ------------------------------
    // Static schedule: this warp alone reads the partition's block-table
    // slice, so the first copies go out without waiting for the compute
    // warps' prologue (with spec_table the slice is already in smem: same
    // start, same lanes).  Work list: the unit's CTAs claim its 64-token
    // stages from an epoch-tagged counter in the workspace, the first claim a
    // ring's worth, later claims one stage, each issued a stage ahead; the
    // copy warp reads each claimed stage's block-table entries itself.
    // The work list also passes each stage's first token through s_c0 before
    // the stage's arrival, and a last stage with s_c0 = -1 tells the compute
    // warps to stop (the static schedule's warps count its stages).
    if constexpr (!WL) {
      for (int i = lane; i < nbt; i += 32) {
        int phys =
            spec_table ? bt_s[i] : a.block_tables[(size_t)b * a.max_blocks_per_seq + jb0 + i];
        if (phys < 0 || phys >= a.num_blocks) {
          atomicOr(&g_pa_status, PA_DEV_BAD_BLOCK);
          phys = -1;
        }
        bt_s[i] = phys;
      }
    }
    __syncwarp();
    const int nbox = TS / BR;
    const int nitem = nbox * 2;  // (box, K/V) per lane
    const int nst_unit = (S - A + TS - 1) / TS;
    // Work list: s_j is the j-th stage this CTA copies.  At iteration j the
    // numbers of s_j .. s_j+2 are known (st_cur, st_n1, st_n2) and this lane's
    // block-table entry for s_j was read at the end of iteration j - 2 into
    // the register of j's parity (rawA / rawB); claims alternate between two
    // in-flight atomics (pendA / pendB) the same way.  Values still in
    // flight are never copied between registers, so no wait lands on an
    // iteration earlier than the one that uses the value.
    int st_cur = 0, st_n1 = 0, st_n2 = 0;
    int rawA = 0, rawB = 0;
    unsigned long long pendA = 0, pendB = 0;  // lane 0
    int run = 0, run_left = 0;  // this CTA's fixed stages not yet taken: run, run + 1, ...
    constexpr int kNoBox = INT_MIN;
    // This lane's block-table entry for stage st (kNoBox: nothing to copy).
    auto table_entry = [&](int st) -> int {
      if (st >= nst_unit || lane >= nitem) return kNoBox;
      const int bt0 = A + st * TS + (lane >> 1) * BR;
      if (bt0 >= S || bt0 + BR <= ulo) return kNoBox;
      return a.block_tables[(size_t)b * a.max_blocks_per_seq + (bt0 >> a.block_shift)];
    };
    constexpr int kFixed = NSTAGE + 2;  // work list: stages each CTA owns outright
    unsigned long long seen_ctr = 0, seen_done = 0;  // lane 0: the counters as first read
    unsigned long long* ctr = a.stage_ctr + (size_t)blockIdx.z * gridDim.y + blockIdx.y;
    unsigned long long* done = a.done + (size_t)blockIdx.z * gridDim.y + blockIdx.y;
    if constexpr (WL) {
      // A ring's worth plus two stages per CTA are fixed (CTA `part` starts
      // at stage part * kFixed), so the first copies wait for no claim; later
      // stages come from the unit's counter, numbered past all the fixed
      // ones.  The counters are read now and reset (if stale) after stage
      // 0's copies; claims are resolved three stages ahead and block-table
      // entries read two ahead, each waited for after a stage's copies are
      // out, and the unit's block-table lines are prefetched into L2, spread
      // over its CTAs.
      if (lane == 0) {
        seen_ctr = ld_relaxed_u64(ctr);
        seen_done = ld_relaxed_u64(done);
      }
      const int* tb = a.block_tables + (size_t)b * a.max_blocks_per_seq;
      const int e1 = ((S - 1) >> a.block_shift) + 1;
      for (int e = ((A >> a.block_shift) & ~31) + (part * 32 + lane) * 32; e < e1;
           e += nparts * 32 * 32)
        prefetch_l2(tb + e);
      st_cur = min(part * kFixed, nst_unit);
      st_n1 = min(st_cur + 1, nst_unit);
      st_n2 = min(st_cur + 2, nst_unit);
      run = st_cur + 3;
      run_left = kFixed - 3;
      rawA = table_entry(st_cur);
      rawB = table_entry(st_n1);
    }
    const int dyn0 = nparts * kFixed;  // first stage handed out by the counter

    const uint64_t kv_policy = l2_evict_first_policy();  // K/V are read once
    // Copies stage number kk (ring slot kk % NSTAGE) of tokens [c0, c0 + TS);
    // raw: the work list's block-table entry for this lane's box.  False if
    // the wait for the slot timed out.
    auto issue = [&](int kk, int c0, int raw) -> bool {
      const int s = kk % NSTAGE;
      if (kk >= NSTAGE) {
        bool got = true;
        if (lane == 0) got = mbar_wait(smem_u32(&bars[NSTAGE + s]), ((kk / NSTAGE) - 1) & 1);
        if (!__shfl_sync(FULL, got, 0)) return false;
      }
      const int ta = max(c0, ulo), te = min(c0 + TS, p1);
      bool mine = false;
      uint32_t dst = 0;
      int y = 0, isv = 0;
      if (lane < nitem) {
        const int j = lane >> 1;
        isv = lane & 1;
        const int bt0 = c0 + j * BR;
        if (bt0 + BR > ta && bt0 < te) {
          const int jj = bt0 >> a.block_shift;
          int phys;
          if constexpr (WL) {
            phys = raw;
            if (phys < 0 || phys >= a.num_blocks) {
              atomicOr(&g_pa_status, PA_DEV_BAD_BLOCK);
              phys = -1;
            }
          } else {
            phys = bt_s[jj - jb0];
          }
          if (phys >= 0) {
            mine = true;
            y = (phys * a.num_kv_heads + kvh) * a.block_size + (bt0 - (jj << a.block_shift));
            dst = s * T::STAGE_BYTES + isv * T::KV_BYTES + j * box_bytes;
          }
        }
      }
      // self-refill: boxes of the stage's second half complete its own barrier
      const bool hi = selfref && lane < nitem && (lane >> 1) * BR >= TS / 2;
      const uint32_t all = __ballot_sync(FULL, mine), high = __ballot_sync(FULL, mine && hi);
      if (lane == 0) {
        if constexpr (WL) s_c0[s] = c0;
        mbar_arrive_expect_tx(smem_u32(&bars[s]), __popc(all & ~high) * box_bytes);
        if (selfref) mbar_arrive_expect_tx(smem_u32(&bars[NSTAGE + s]), __popc(high) * box_bytes);
      }
      __syncwarp();
      if (mine)
        tma_load_3d_hint(smem_u32(smem) + dst,
                         isv ? static_cast<const void*>(&tmv) : static_cast<const void*>(&tmk), 0,
                         y, 0, smem_u32(&bars[hi ? NSTAGE + s : s]), kv_policy);
      return true;
    };
    // Work list, after stage kk's copies: the next stage numbers, the claim
    // of kk's parity, and the block-table read for stage kk + 2 (same parity).
    auto advance = [&](int kk, unsigned long long& pend, int& raw) {
      if (kk == 0 && lane == 0) {  // open this CTA's claims
        epoch_reset_if_stale(ctr, seen_ctr, a.epoch);
        // Claims must resolve in the order their tickets were taken, so that
        // a CTA's first out-of-range ticket comes after all its valid ones
        // (the copies stop there).  The first claim resolves at stage
        // kFixed - 3, on that stage's parity: the lower ticket goes there.
        const unsigned long long t0 = atomicAdd(ctr, 1ull);
        const unsigned long long t1 = atomicAdd(ctr, 1ull);
        if constexpr (((kFixed - 3) & 1) == 0) {
          pendA = t0;
          pendB = t1;
        } else {
          pendB = t0;
          pendA = t1;
        }
        epoch_reset_if_stale(done, seen_done, a.epoch);
        s_dtouch = 1;
      }
      int st_n3;
      if (run_left > 0) {
        st_n3 = min(run++, nst_unit);
        --run_left;
      } else {
        int v = 0;
        if (lane == 0) {
          v = claim_value(pend, a.epoch);  // INT_MAX (stop) if not this call's
          v = v >= nst_unit - dyn0 ? nst_unit : dyn0 + v;
          pend = atomicAdd(ctr, 1ull);
        }
        st_n3 = __shfl_sync(FULL, v, 0);
      }
      st_cur = st_n1;
      st_n1 = st_n2;
      st_n2 = st_n3;
      raw = table_entry(st_n1);
    };

    int k = spec0 ? 1 : 0;
    bool ok = true;
    if constexpr (!WL) {
      // self-refill: the first ring's worth only; the compute warps refill
      const int kcopy = selfref ? min(nst, NSTAGE) : nst;
      for (; k < kcopy; ++k)
        if (!issue(k, p0 + k * TS, 0)) {
          ok = false;
          break;
        }
    } else {
      for (;; k += 2) {
        if (st_cur >= nst_unit) break;
        if (!issue(k, A + st_cur * TS, rawA)) {
          ok = false;
          break;
        }
        advance(k, pendA, rawA);
        if (st_cur >= nst_unit) {
          k += 1;
          break;
        }
        if (!issue(k + 1, A + st_cur * TS, rawB)) {
          k += 1;
          ok = false;
          break;
        }
        advance(k + 1, pendB, rawB);
      }
    }
    const int issued = k;
    if (WL && ok && lane == 0) {
      // the stop stage: its slot last held stage issued - NSTAGE
      const int s = issued % NSTAGE;
      bool got = true;
      if (issued >= NSTAGE) got = mbar_wait(smem_u32(&bars[NSTAGE + s]), ((issued / NSTAGE) - 1) & 1);
      if (got) {
        s_c0[s] = -1;
        mbar_arrive(smem_u32(&bars[s]));
      }
    }
    // (self-refill: the compute warps wait for every stage this warp issued)
    if (lane == 0 && !selfref) {
      for (int kk = max(0, issued - NSTAGE + (WL ? 1 : 0)); kk < issued; ++kk)
        mbar_wait(smem_u32(&bars[kk % NSTAGE]), (kk / NSTAGE) & 1);
    }
    __syncwarp();
  } else {
    // ----------------------------- compute warps ---------------------------
    const int cw = warp - 1;
    const int rt = cw % NRT;
    const int slice = cw / NRT;
    const int nslice = (NCW - 1 - rt) / NRT + 1;
    const int quad = lane >> 2, qi = lane & 3;
    qoff = row_token_offset(a.query_lens, b, lane);
    if (warp == 1 && lane == 0) s_qoff = qoff;  // for the copy warp's share of the merge
    const int brs = 31 - __clz(BR);  // log2(BR)
    // lane parts of the ldmatrix row addresses (token row within the chunk,
    // 16-byte chunk parity) for K (A operand) and V (A operand, transposed)
    const int lt_k = (((lane >> 3) & 1) << 3) + (lane & 7), ck_k = lane >> 4;
    // (FP8 V uses the K addresses: its x4 covers tokens 0-7 / 8-15 of two chunks.)
    const int lt_v = F8 ? lt_k : ((lane >> 4) << 3) + (lane & 7);
    const int ck_v = F8 ? ck_k : (lane >> 3) & 1;
    const uint32_t kofs = box_lane_off<T::BOXW>(lt_k, ck_k);
    const uint32_t vofs = box_lane_off<T::BOXW>(lt_v, ck_v);
    const uint32_t half = (uint32_t)BR * 128u;
    int lo_max, hi_min, dummy;
    query_range(S, L, L - 1, w, lo_max, dummy);  // the last token sees the latest start
    query_range(S, L, 0, w, dummy, hi_min);      // the first token sees the earliest end

    // Q^T as B fragments: n-tile n holds warp-tile rows n*8..n*8+7; this
    // thread feeds row n*8 + quad, dims ks*16 + 2*qi (+1) and +8 (+9) (bf16
    // caches), or dims ks*16 + 4*qi .. +3 (FP8 caches, f16 operands).
    uint32_t qb[T::KSTEPS][N8][2];
    // Softmax statistics of the rows n*8 + 2*qi + j (j = 0, 1): the O^T columns
    // this thread accumulates.
    int lo_r[N8][2], hi_r[N8][2];
#pragma unroll
    for (int n = 0; n < N8; ++n) {
      const int rq = rt * RT + n * 8 + quad;
      size_t qrow = 0;
      const bool has_q = rq < Rs;
      if (has_q) {
        const int rr = row0 + rq;
        const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
        qrow = ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D;
      }
#pragma unroll
      for (int ks = 0; ks < T::KSTEPS; ++ks) {
        uint32_t b0 = 0u, b1 = 0u;
        if (has_q) {
          if constexpr (F8) {
            if (a.q_fp8) {
              const uint32_t w4 = __ldg(reinterpret_cast<const uint32_t*>(a.q8 + qrow) + ks * 4 + qi);
              b0 = e4m3x2_to_f16x2(w4 & 0xffffu);
              b1 = e4m3x2_to_f16x2(w4 >> 16);
            } else {
              const uint2 w4 = __ldg(reinterpret_cast<const uint2*>(a.q + qrow) + ks * 4 + qi);
              b0 = bf16x2_to_f16x2(w4.x);
              b1 = bf16x2_to_f16x2(w4.y);
            }
          } else {
            if (a.q_fp8) {
              const unsigned short* qp = reinterpret_cast<const unsigned short*>(a.q8 + qrow);
              b0 = f16x2_to_bf16x2(e4m3x2_to_f16x2(__ldg(qp + ks * 8 + qi)));
              b1 = f16x2_to_bf16x2(e4m3x2_to_f16x2(__ldg(qp + ks * 8 + qi + 4)));
            } else {
              const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q + qrow);
              b0 = __ldg(qp + ks * 8 + qi);
              b1 = __ldg(qp + ks * 8 + qi + 4);
            }
          }
        }
        qb[ks][n][0] = b0;
        qb[ks][n][1] = b1;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rs = rt * RT + n * 8 + 2 * qi + j;
        lo_r[n][j] = INT_MAX;
        hi_r[n][j] = INT_MIN;
        if (rs < Rs) query_range(S, L, (row0 + rs) / a.group, w, lo_r[n][j], hi_r[n][j]);
      }
    }

    float o[T::MD][N8][4];
#pragma unroll
    for (int md = 0; md < T::MD; ++md)
#pragma unroll
      for (int n = 0; n < N8; ++n) o[md][n][0] = o[md][n][1] = o[md][n][2] = o[md][n][3] = 0.f;
    float m_r[N8][2], l_r[N8][2];
#pragma unroll
    for (int n = 0; n < N8; ++n) m_r[n][0] = m_r[n][1] = kNegInf, l_r[n][0] = l_r[n][1] = 0.f;

    // Chunks of 16 tokens, NCH at a time: the scores of all NCH chunks, one
    // online-softmax update over them, then their PV products.  With NCH = 2
    // a warp carries two independent MMA chains through each phase.
    auto process = [&](auto nch_c, int ch_first, int ch_step, int c0, uint32_t Ks, uint32_t Vs,
                       bool all_valid, bool boundary) {
      constexpr int NCH = decltype(nch_c)::value;
      // S^T = K Q^T; a single chunk with one n-tile uses two accumulator sets
      // (even / odd d steps) to halve the dependent MMA chain.
      constexpr int NACC = (NCH == 1 && N8 == 1) ? 2 : 1;
      int tbs[NCH];
      uint32_t cbs[NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tbs[c] = (ch_first + c * ch_step) * 16;
        // the chunk's 16 tokens lie in one box (BR >= 16)
        cbs[c] = (uint32_t)((tbs[c] >> brs) * box_bytes + (tbs[c] & (BR - 1)) * T::BOXW);
      }
      float sc[NCH][NACC][N8][4];
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int u = 0; u < NACC; ++u)
#pragma unroll
          for (int n = 0; n < N8; ++n)
            sc[c][u][n][0] = sc[c][u][n][1] = sc[c][u][n][2] = sc[c][u][n][3] = 0.f;
      if constexpr (F8) {
        // one x4 = tokens 0-7 / 8-15 of chunks 2kp, 2kp+1: two k-steps
#pragma unroll
        for (int kp = 0; kp < T::KSTEPS / 2; ++kp) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            uint32_t r[4];
            ldsm_x4(Ks + cbs[c] + box_step_off<T::BOXW>(kp, kofs, half), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t ka[4];
              e4m3x4_to_f16x2x2(r[2 * h], ka[0], ka[2]);
              e4m3x4_to_f16x2x2(r[2 * h + 1], ka[1], ka[3]);
              const int ks = 2 * kp + h;
#pragma unroll
              for (int n = 0; n < N8; ++n)
                mma_f16_16816(sc[c][ks % NACC][n], ka, qb[ks][n][0], qb[ks][n][1]);
            }
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < T::KSTEPS; ++ks) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            uint32_t ka[4];
            ldsm_x4(Ks + cbs[c] + box_step_off<T::BOXW>(ks, kofs, half), ka[0], ka[1], ka[2],
                    ka[3]);
#pragma unroll
            for (int n = 0; n < N8; ++n)
              mma_bf16_16816(sc[c][ks % NACC][n], ka, qb[ks][n][0], qb[ks][n][1]);
          }
        }
      }
      // element e of n-tile n: token tb + quad + 8*(e>>1), row n*8 + 2*qi + (e&1)
      float p[NCH][N8][4];
      bool any_rescale = false;
      float al[N8][2];
#pragma unroll
      for (int n = 0; n < N8; ++n) {
        float v[NCH][4];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float x = sc[c][0][n][e];
            if constexpr (NACC == 2) x += sc[c][1][n][e];
            v[c][e] = x * a.scale_log2;
          }
          if (!all_valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t = c0 + tbs[c] + quad + ((e >> 1) << 3);
              v[c][e] = (t >= lo_r[n][e & 1] && t < hi_r[n][e & 1]) ? v[c][e] : kNegInf;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = fmaxf(v[0][j], v[0][j + 2]);
#pragma unroll
          for (int c = 1; c < NCH; ++c) mx = fmaxf(mx, fmaxf(v[c][j], v[c][j + 2]));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
          // The running maximum moves only when the chunks' maximum passes it
          // by more than kLazyMax (log2 units): probabilities stay below
          // 2^kLazyMax, and after the first chunks O is rarely rescaled.
          const bool up = mx > m_r[n][j] + kLazyMax;  // m_r = -inf: any finite mx
          const float mn = up ? mx : m_r[n][j];
          const float mu = (mn == kNegInf) ? 0.f : mn;
          al[n][j] = up ? ex2(m_r[n][j] - mu) : 1.f;  // first update: 2^-inf = 0 (O, l are 0)
          any_rescale |= up;
          m_r[n][j] = mn;
          float ps = 0.f;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            p[c][n][j] = ex2(v[c][j] - mu);
            p[c][n][j + 2] = ex2(v[c][j + 2] - mu);
            ps += p[c][n][j] + p[c][n][j + 2];
          }
          l_r[n][j] = l_r[n][j] * al[n][j] + ps;
        }
      }
      if (__any_sync(FULL, any_rescale)) {
#pragma unroll
        for (int md = 0; md < T::MD; ++md)
#pragma unroll
          for (int n = 0; n < N8; ++n) {
            o[md][n][0] *= al[n][0];
            o[md][n][1] *= al[n][1];
            o[md][n][2] *= al[n][0];
            o[md][n][3] *= al[n][1];
          }
      }
      // P^T B fragments: the accumulator's 8x8 blocks transposed in registers.
      uint32_t pb[NCH][N8][2];
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int n = 0; n < N8; ++n) {
          if constexpr (F8) {
            pb[c][n][0] = movmatrix_trans(pack_f16x2(p[c][n][0], p[c][n][1]));
            pb[c][n][1] = movmatrix_trans(pack_f16x2(p[c][n][2], p[c][n][3]));
          } else {
            pb[c][n][0] = movmatrix_trans(pack_bf16x2(p[c][n][0], p[c][n][1]));
            pb[c][n][1] = movmatrix_trans(pack_bf16x2(p[c][n][2], p[c][n][3]));
          }
        }
      uint32_t mk_lo[NCH], mk_hi[NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        mk_lo[c] = mk_hi[c] = 0xffffffffu;
        if (boundary) {
          const int t = c0 + tbs[c] + 2 * qi;
          auto in = [&](int u) { return u >= ulo && u < p1; };
          mk_lo[c] = (in(t) ? 0x0000ffffu : 0u) | (in(t + 1) ? 0xffff0000u : 0u);
          mk_hi[c] = (in(t + 8) ? 0x0000ffffu : 0u) | (in(t + 9) ? 0xffff0000u : 0u);
        }
      }
      // O^T += V^T P^T; the V lanes of tokens outside [ulo, p1) are zeroed
      // only in stages that reach past those bounds (masked = true).
      auto pv = [&](auto masked) {
        constexpr bool MK = decltype(masked)::value;
        if constexpr (F8) {
          // one x4.trans = tokens 0-7 / 8-15 of chunks 2mp, 2mp+1: two M
          // tiles; a register holds dims (2g, 2g+1) of tokens (2c, 2c+1),
          // regrouped by dim before the conversion (masks act on f16 halves)
#pragma unroll
          for (int mp = 0; mp < T::MD / 2; ++mp) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              uint32_t r[4];
              ldsm_x4_t(Vs + cbs[c] + box_step_off<T::BOXW>(mp, vofs, half), r[0], r[1], r[2],
                        r[3]);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t va[4];
                e4m3x4_to_f16x2x2(__byte_perm(r[2 * h], 0, 0x3120), va[0], va[1]);
                e4m3x4_to_f16x2x2(__byte_perm(r[2 * h + 1], 0, 0x3120), va[2], va[3]);
                if constexpr (MK) {
                  va[0] &= mk_lo[c];
                  va[1] &= mk_lo[c];
                  va[2] &= mk_hi[c];
                  va[3] &= mk_hi[c];
                }
#pragma unroll
                for (int n = 0; n < N8; ++n)
                  mma_f16_16816(o[2 * mp + h][n], va, pb[c][n][0], pb[c][n][1]);
              }
            }
          }
        } else {
#pragma unroll
          for (int md = 0; md < T::MD; ++md) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              uint32_t va[4];
              ldsm_x4_t(Vs + cbs[c] + box_step_off<T::BOXW>(md, vofs, half), va[0], va[1],
                        va[2], va[3]);
              if constexpr (MK) {
                va[0] &= mk_lo[c];
                va[1] &= mk_lo[c];
                va[2] &= mk_hi[c];
                va[3] &= mk_hi[c];
              }
#pragma unroll
              for (int n = 0; n < N8; ++n) mma_bf16_16816(o[md][n], va, pb[c][n][0], pb[c][n][1]);
            }
          }
        }
      };
      if (boundary)
        pv(std::true_type{});
      else
        pv(std::false_type{});
    };

    // Paired mode (FP8 caches, units of at most 8 rows, an even ring depth):
    // warps 1-2 consume the even stages and warps 3-4 the odd ones, each warp
    // two chunks (one 32-token half) of its stage at once, so each warp
    // carries two MMA chains, and each ring slot always serves the same two
    // warps (a parity wait never skips one of its phases).  With self-refill
    // each warp also refills its own half of the slot with the stage NSTAGE
    // ahead as soon as it has read it: the copy warp, which issues a stage's 8
    // box requests one after another, would otherwise sit between every
    // release and the next copy.  Each half then has its own full barrier,
    // waited for and re-armed by that one warp.  Every other case: every
    // compute warp consumes every stage, its chunks one by one, and the copy
    // warp refills the ring.
    const int kfirst = paired ? (slice >> 1) : 0;
    const int kstep = paired ? 2 : 1;
    const int kend = WL ? INT_MAX : nst;
    const int hsel = slice & 1;  // paired mode: this warp's half of its stages
    const uint64_t kv_policy_c = l2_evict_first_policy();
    // Self-refill: copies this warp's half of stage kk into slot s (barrier fb).
    auto refill = [&](int kk, int s, uint32_t fb) {
      fence_proxy_async_smem();  // this warp's reads of the half, before the copies overwrite it
      const int hs = p0 + kk * TS + hsel * (TS / 2);  // the half's first token
      const int ta = max(hs, ulo), te = min(hs + TS / 2, p1);
      const int nb = (TS / 2) / BR;  // boxes per half
      bool mine = false;
      uint32_t dst = 0;
      int y = 0, isv = 0;
      if (lane < 2 * nb) {
        const int j = lane >> 1;
        isv = lane & 1;
        const int bt0 = hs + j * BR;
        if (bt0 + BR > ta && bt0 < te) {
          const int jj = bt0 >> a.block_shift;
          const int phys = bt_s[jj - jb0];
          if (phys >= 0) {
            mine = true;
            y = (phys * a.num_kv_heads + kvh) * a.block_size + (bt0 - (jj << a.block_shift));
            dst = s * T::STAGE_BYTES + isv * T::KV_BYTES + (hsel * nb + j) * box_bytes;
          }
        }
      }
      const uint32_t nload = __popc(__ballot_sync(FULL, mine));
      if (lane == 0) mbar_arrive_expect_tx(fb, nload * box_bytes);
      __syncwarp();
      if (mine)
        tma_load_3d_hint(smem_u32(smem) + dst,
                         isv ? static_cast<const void*>(&tmv) : static_cast<const void*>(&tmk), 0,
                         y, 0, fb, kv_policy_c);
    };
    int kgave = -1;  // self-refill: the stage whose wait gave up
    for (int k = kfirst; k < kend; k += kstep) {
      const int s = k % NSTAGE;
      const uint32_t fb = smem_u32(&bars[(selfref && hsel) ? NSTAGE + s : s]);
      const bool got = mbar_wait(fb, (k / NSTAGE) & 1);
      if (!__all_sync(FULL, got)) {
        kgave = k;
        break;
      }
      int c0 = p0 + k * TS;
      if constexpr (WL) {
        c0 = s_c0[s];
        if (c0 < 0) break;
      }
      const uint32_t Ks = smem_u32(smem + s * T::STAGE_BYTES);
      const uint32_t Vs = Ks + T::KV_BYTES;
      const bool all_valid = (c0 >= lo_max) && (c0 + TS <= hi_min);
      const bool boundary = (c0 < ulo) || (c0 + TS > p1);
      if constexpr (PAIRABLE) {
        if (paired) {
          process(std::integral_constant<int, 2>{}, 2 * (slice & 1), 1, c0, Ks, Vs, all_valid,
                  boundary);
        } else {
          for (int ch = slice; ch < TS / 16; ch += nslice)
            process(std::integral_constant<int, 1>{}, ch, 0, c0, Ks, Vs, all_valid, boundary);
        }
      } else {
        for (int ch = slice; ch < TS / 16; ch += nslice)
          process(std::integral_constant<int, 1>{}, ch, 0, c0, Ks, Vs, all_valid, boundary);
      }
      __syncwarp();
      if (selfref) {
        if (k + NSTAGE < kend) refill(k + NSTAGE, s, fb);
      } else if (lane == 0) {
        mbar_arrive(smem_u32(&bars[NSTAGE + s]));
      }
    }
    if (selfref && kgave >= 0 && lane == 0) {
      // A wait gave up (the status is set): this warp's copies still in
      // flight, the stage it waited for and the next one of its slots, land
      // (bounded waits) before the CTA can leave.
      for (int kk = kgave; kk < kend && kk <= kgave + 2; kk += 2)
        mbar_wait(smem_u32(&bars[hsel ? NSTAGE + kk % NSTAGE : kk % NSTAGE]), (kk / NSTAGE) & 1);
    }

    named_bar_sync(1, NCW * 32);
    if constexpr (F8) {
      // O^T element (md, n, e): dim md*16 + 2*quad + (e>>1), row n*8 + 2*qi + (e&1)
#pragma unroll
      for (int md = 0; md < T::MD; ++md)
#pragma unroll
        for (int n = 0; n < N8; ++n)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            *reinterpret_cast<float2*>(
                &comb_acc[(cw * RT + n * 8 + 2 * qi + j) * C::LD + md * 16 + 2 * quad]) =
                make_float2(o[md][n][j], o[md][n][j + 2]);
    } else {
      // O^T element (md, n, e): dim md*16 + quad + 8*(e>>1), row n*8 + 2*qi + (e&1)
#pragma unroll
      for (int md = 0; md < T::MD; ++md)
#pragma unroll
        for (int n = 0; n < N8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            comb_acc[(cw * RT + n * 8 + 2 * qi + (e & 1)) * C::LD + md * 16 + quad +
                     ((e >> 1) << 3)] = o[md][n][e];
    }
#pragma unroll
    for (int n = 0; n < N8; ++n)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float l = l_r[n][j];
        l += __shfl_xor_sync(FULL, l, 4);
        l += __shfl_xor_sync(FULL, l, 8);
        l += __shfl_xor_sync(FULL, l, 16);
        if (quad == 0) {
          comb_l[cw * RT + n * 8 + 2 * qi + j] = l;
          comb_m[cw * RT + n * 8 + 2 * qi + j] = m_r[n][j];
        }
      }
  }
  __syncthreads();
  if (warp == 0) qoff = s_qoff;

  // ----------------- merge the compute warps' partials --------------------
  // Per row: the slices' common max M, each slice's factor 2^(m_c - M) and
  // the sum Z; then every float4 column is an independent weighted sum.
  for (int r = threadIdx.x; r < Rs; r += blockDim.x) {
    const int rti = r / RT, rr8 = r - (r / RT) * RT;
    float M = kNegInf;
    for (int c = rti; c < NCW; c += NRT) M = fmaxf(M, comb_m[c * RT + rr8]);
    float Z = 0.f;
    for (int c = rti; c < NCW; c += NRT) {
      const float f = (M == kNegInf) ? 0.f : ex2(comb_m[c * RT + rr8] - M);
      s_fac[c][r] = f;
      Z += f * comb_l[c * RT + rr8];
    }
    s_rowm[r] = M;
    s_rowz[r] = Z;
  }
  __syncthreads();
  constexpr int C4 = D / 4;
  for (int it = threadIdx.x; it < Rs * C4; it += blockDim.x) {
    const int r = it / C4, c4 = it - (it / C4) * C4;
    const int rti = r / RT, rr8 = r - (r / RT) * RT;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = rti; c < NCW; c += NRT) {
      const float f = s_fac[c][r];
      const float4 v = *reinterpret_cast<const float4*>(comb_acc + (c * RT + rr8) * C::LD + c4 * 4);
      acc.x += f * v.x;
      acc.y += f * v.y;
      acc.z += f * v.z;
      acc.w += f * v.w;
    }
    const float Z = s_rowz[r];
    const int rr = row0 + r;
    if (nparts == 1) {
      const float inv = a.v_scale / Z;
      const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
      __nv_bfloat16* dp =
          a.dst + ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + c4 * 4;
      // one 8-byte store per lane: a warp writes whole 32-byte sectors
      *reinterpret_cast<uint2*>(dp) = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv),
                                                 pack_bf16x2(acc.z * inv, acc.w * inv));
    } else {
      const float inv = Z > 0.f ? a.v_scale / Z : 0.f;
      const size_t base =
          ((size_t)(b * a.num_kv_heads + kvh) * a.max_parts + part) * a.max_rows + rr;
      *reinterpret_cast<float4*>(a.ws_o + base * D + c4 * 4) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      if (c4 == 0) a.ws_lse[base] = Z > 0.f ? s_rowm[r] + lg2(Z) : kNegInf;
    }
  }
  if constexpr (WL)
    if (nparts > 1) merge_unit_partials<D>(a, b, kvh, part, nparts, row0, Rs, qoff, s_dtouch);
}

// ---------------------------------------------------------------------------
// Log-sum-exp reduce (ExecuTorch PR #18759, the split-K reduce kernel):
// per (row, kv head, batch row): M = max_p lse_p, w_p = 2^(lse_p - M),
// dst = sum_p w_p O_p / sum_p w_p.  Partials are normalised, so the weights
// carry each partition's softmax mass.
//
// One CTA per (row, kv head, batch row) and DSPLIT-th of head_dim.  A
// partial's slice of DC dims is LPP = DC/4 lanes (one float4 each), so a warp
// covers PPW = 32/LPP partials per load; the CTA's warps share the partials
// so that a lane holds at most two of them per round, and its loads are
// issued together before it merges them: one L2 round trip, whatever the
// register allocator makes of the code.  (A deeper per-lane batch of eight
// was compiled into a few dependent rounds at a low register count: several
// L2 round trips for the hundreds of partials of a long row; this takes one.)
// Lanes keep a running (max, sum, weighted sum); lanes of a warp, then the
// warps (through shared memory, merged as a tree by warp 0), combine with the
// same rescale.  Rows with many partials split head_dim over more CTAs so
// that 16 warps suffice and more SMs pull partials from L2.
//
// Launched with programmatic stream serialization: it is scheduled while the
// partition kernel drains.  The lengths, windows and the row's q offset are
// read before griddepcontrol.wait: they are inputs of the call, which the
// partition kernel reads too, and it triggers this launch only after its own
// griddepcontrol.wait, so whatever wrote them has completed.  Only the
// partials are read after the wait.
// ---------------------------------------------------------------------------
template <int D, int DSPLIT>
__global__ void __launch_bounds__(1024) pa_reduce_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int DC = D / DSPLIT;  // dims per CTA
  constexpr int LPP = DC / 4;     // lanes per partial slice (one float4 each)
  constexpr int PPW = 32 / LPP;   // partials per warp load
  static_assert(LPP >= 1 && LPP <= 32, "a partial's slice must fit a warp");
  __shared__ float s_m[32][LPP], s_z[32][LPP];
  __shared__ float4 s_o[32][LPP];
  __shared__ int s_qoff;

  // The next call's partition kernel may launch now: its CTAs take the SMs
  // the partition grid leaves, set up and prefetch while this grid works,
  // and wait for its completion before reading any input.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int rr = blockIdx.x / DSPLIT, ch = blockIdx.x - (blockIdx.x / DSPLIT) * DSPLIT;
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  if (warp == 0) {
    const int q0 = row_token_offset(a.query_lens, b, lane);
    if (lane == 0) s_qoff = q0;
  }
  const int S = a.seq_lens[b];
  const int L = a.query_lens[b];
  const int w = a.windows ? a.windows[b] : a.window;
  if (L <= 0 || L > S || w < 0 || S > a.max_blocks_per_seq * a.block_size) return;
  const int R = a.group * L;
  if (rr >= R || R > a.max_rows) return;
  const int A = union_lo(S, L, w) & ~(kStageTokens - 1);
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (nparts <= 1 || nparts > a.max_parts) return;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials are complete

  const int sub = lane / LPP, c4 = lane - (lane / LPP) * LPP;
  const size_t ubase = (size_t)(b * a.num_kv_heads + kvh) * a.max_parts;
  const float* lse = a.ws_lse + ubase * a.max_rows + rr;
  const float4* ob =
      reinterpret_cast<const float4*>(a.ws_o + (ubase * a.max_rows + rr) * D + ch * DC) + c4;
  const size_t pst4 = (size_t)a.max_rows * D / 4;  // float4 stride between partials
  const int step = nw * PPW;
  LseAcc acc{kNegInf, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
  for (int p0 = warp * PPW + sub; p0 < nparts; p0 += 2 * step) {
    const int p1 = p0 + step;
    const float l0 = lse[(size_t)p0 * a.max_rows];
    const float4 o0 = ob[(size_t)p0 * pst4];
    float l1 = kNegInf;
    float4 o1 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p1 < nparts) {
      l1 = lse[(size_t)p1 * a.max_rows];
      o1 = ob[(size_t)p1 * pst4];
    }
    lse_merge(acc, l0, 1.f, o0);
    lse_merge(acc, l1, 1.f, o1);
  }
  // lanes holding the same dims (c4) in other slices of the warp
#pragma unroll
  for (int off = LPP; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(FULL, acc.m, off);
    const float z2 = __shfl_xor_sync(FULL, acc.z, off);
    float4 o2;
    o2.x = __shfl_xor_sync(FULL, acc.o.x, off);
    o2.y = __shfl_xor_sync(FULL, acc.o.y, off);
    o2.z = __shfl_xor_sync(FULL, acc.o.z, off);
    o2.w = __shfl_xor_sync(FULL, acc.o.w, off);
    lse_merge(acc, m2, z2, o2);
  }
  if (sub == 0) {
    s_o[warp][c4] = acc.o;
    s_m[warp][c4] = acc.m;
    s_z[warp][c4] = acc.z;
  }
  __syncthreads();
  if (warp == 0) {
    // warps' results as a tree: lane (g, c4) folds warps g, g + PPW, ...,
    // then the PPW groups of each c4 combine by shuffles
    LseAcc t{kNegInf, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int i = sub; i < nw; i += PPW) lse_merge(t, s_m[i][c4], s_z[i][c4], s_o[i][c4]);
#pragma unroll
    for (int off = LPP; off < 32; off <<= 1) {
      const float m2 = __shfl_xor_sync(FULL, t.m, off);
      const float z2 = __shfl_xor_sync(FULL, t.z, off);
      float4 o2;
      o2.x = __shfl_xor_sync(FULL, t.o.x, off);
      o2.y = __shfl_xor_sync(FULL, t.o.y, off);
      o2.z = __shfl_xor_sync(FULL, t.o.z, off);
      o2.w = __shfl_xor_sync(FULL, t.o.w, off);
      lse_merge(t, m2, z2, o2);
    }
    if (sub == 0) {
      const float inv = t.z > 0.f ? 1.f / t.z : 0.f;
      const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
      __nv_bfloat16* dp = a.dst +
                          ((size_t)(s_qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D +
                          ch * DC + c4 * 4;
      // one 8-byte store per lane: a warp writes whole 32-byte sectors (and
      // whole write requests when dst is mapped host memory)
      *reinterpret_cast<uint2*>(dp) = make_uint2(pack_bf16x2(t.o.x * inv, t.o.y * inv),
                                                 pack_bf16x2(t.o.z * inv, t.o.w * inv));
    }
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

// ---------------------------------------------------------------------------
// Staging copies of the host-buffer entry point.  Each copy owns a run of
// CTAs; a thread issues up to four loads before its stores, so a CTA keeps
// 256 x 4 pieces in flight across the host link.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pa_stage_kernel(const __grid_constant__ StageArgs s) {
  // The partition kernel may launch now: it waits on griddepcontrol for this
  // grid's completion (and its writes) before reading any input.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int c = 0;
  while (c + 1 < s.n && (int)blockIdx.x >= s.c[c + 1].first_block) ++c;
  const StageCopy& sc = s.c[c];
  const int nb = (c + 1 < s.n ? s.c[c + 1].first_block : s.blocks) - sc.first_block;
  const unsigned long long stride = (unsigned long long)nb * blockDim.x;
  const unsigned long long t =
      (unsigned long long)(blockIdx.x - sc.first_block) * blockDim.x + threadIdx.x;
  if (sc.unit == 16) {
    const uint4* src = static_cast<const uint4*>(sc.src);
    uint4* dst = static_cast<uint4*>(sc.dst);
    for (unsigned long long u = t; u < sc.units; u += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (u + j * stride < sc.units) v[j] = src[u + j * stride];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (u + j * stride < sc.units) dst[u + j * stride] = v[j];
    }
  } else if (sc.unit == 4) {
    const uint32_t* src = static_cast<const uint32_t*>(sc.src);
    uint32_t* dst = static_cast<uint32_t*>(sc.dst);
    for (unsigned long long u = t; u < sc.units; u += 4 * stride) {
      uint32_t v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (u + j * stride < sc.units) v[j] = src[u + j * stride];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (u + j * stride < sc.units) dst[u + j * stride] = v[j];
    }
  } else {
    const uint8_t* src = static_cast<const uint8_t*>(sc.src);
    uint8_t* dst = static_cast<uint8_t*>(sc.dst);
    for (unsigned long long u = t; u < sc.units; u += stride) dst[u] = src[u];
  }
}

// Sets a kernel's dynamic-smem limit and asks for the largest shared-memory
// carveout (so two CTAs fit per SM), once per (context, kernel, size): the
// attributes belong to the context, so a context that replaced a reset one
// gets them set again.
cudaError_t ensure_smem_attrs(const void* kern, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<unsigned long long, const void*>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long ctx = context_id();
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({ctx, kern});
  if (ctx != 0 && it != done.end() && it->second >= smem) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  if (ctx != 0) done[{ctx, kern}] = std::max(smem, it != done.end() ? it->second : (size_t)0);
  return cudaSuccess;
}

// Leading blocks of each row that its windowed query tokens (and later ones)
// can no longer see: floor(union_lo / BS).
__global__ void pa_unreachable_kernel(int32_t* count, const int32_t* seq_lens,
                                      const int32_t* query_lens, int window, const int32_t* windows,
                                      int block_shift, int batch) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int S = seq_lens[b], L = query_lens[b];
  const int w = windows ? windows[b] : window;
  int n = 0;
  if (L > 0 && L <= S && w > 0) n = union_lo(S, L, w) >> block_shift;
  if (L > S || L < 0 || w < 0) atomicOr(&g_pa_status, PA_DEV_BAD_ROW);
  count[b] = n;
}

template <int D, int NCW, int NSTAGE>
cudaError_t launch_fma_t(const DecodeArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = pa_partition_fma_kernel<D, NCW, NSTAGE>;
  cudaError_t e = ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 32 * (NCW + 1), smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int NCW, int NSTAGE>
int occupancy_fma_t(size_t smem) {
  auto kern = pa_partition_fma_kernel<D, NCW, NSTAGE>;
  if (ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * (NCW + 1), smem) != cudaSuccess)
    return 0;
  return n;
}

template <int D, int NCW, int NSTAGE, int N8, bool F8>
cudaError_t launch_mma_t(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                         dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = a.worklist ? pa_partition_mma_kernel<D, NCW, NSTAGE, N8, F8, true>
                         : pa_partition_mma_kernel<D, NCW, NSTAGE, N8, F8, false>;
  cudaError_t e = ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // Programmatic stream serialization: CTAs may start (and set up their
  // pipeline) while the previous kernel drains; they wait on griddepcontrol
  // before reading any input.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(32 * (NCW + 1));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;  // work list: every CTA resident at once
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.worklist ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a, tk, tv);
}

template <int D, int NCW, int NSTAGE, int N8, bool F8>
int occupancy_mma_t(size_t smem) {
  auto kern = pa_partition_mma_kernel<D, NCW, NSTAGE, N8, F8, false>;
  if (ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * (NCW + 1), smem) != cudaSuccess)
    return 0;
  return n;
}


#include "pa_tc.cuh"

template <int NS, int RT>
cudaError_t launch_tc_t(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                        dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = pa_partition_tc_kernel<NS, RT>;
  cudaError_t e = ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, tk, tv);
}

// Resident CTAs per SM from the kernel's own limits.  (The runtime's
// occupancy query answers 1 for this kernel at any shared-memory size, while
// two CTAs per SM are observed resident on B200, as shared memory, registers
// and tensor memory allow.)
template <int NS, int RT>
int occupancy_tc_t(size_t smem) {
  auto kern = pa_partition_tc_kernel<NS, RT>;
  if (ensure_smem_attrs(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return 0;
  cudaFuncAttributes fa;
  int dev = 0, sm_smem = 0, sm_regs = 0, reserved = 0;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
          cudaSuccess)
    return 0;
  const long long per_cta_smem = (long long)smem + (long long)fa.sharedSizeBytes + reserved;
  const int regs = ((fa.numRegs + 7) / 8) * 8;  // allocated per thread in units of 8
  int n = (int)(sm_smem / per_cta_smem);
  n = std::min(n, sm_regs / (regs * 320));
  n = std::min(n, 512 / kTcTmemCols);  // tensor-memory columns per SM
  return std::max(n, 0);
}

}  // namespace

size_t tc_smem_bytes(int stages, int part_tokens, int block_size) {
  const size_t nbt = (size_t)part_tokens / block_size + 2;
  return 1024 + (size_t)stages * TcLayout::STAGE_BYTES + 2 * TcLayout::QB_BYTES +
         4 * TcLayout::PB_BYTES + (2 * (size_t)stages + 9) * sizeof(uint64_t) +
         (2 * 4 + 4 + 4 + 1) * kTcN * sizeof(float) + nbt * sizeof(int);
}

cudaError_t launch_partition_tc(const DecodeArgs& a, const KernelShape& k, const CUtensorMap& tk,
                                const CUtensorMap& tv, dim3 grid, size_t smem,
                                cudaStream_t stream) {
  if (k.head_dim == 128 && k.stages == 3 && k.n8 == 1 && k.kv_fp8)
    return launch_tc_t<3, 8>(a, tk, tv, grid, smem, stream);
  return cudaErrorInvalidValue;
}

int occupancy_partition_tc(const KernelShape& k, size_t smem) {
  if (k.head_dim == 128 && k.stages == 3 && k.n8 == 1 && k.kv_fp8) return occupancy_tc_t<3, 8>(smem);
  return 0;
}

size_t mma_smem_bytes(int head_dim, int elem_bytes, int stages, int part_tokens, int block_size) {
  const size_t ring = (size_t)stages * 2 * TS * head_dim * elem_bytes;
  const size_t nbt = (size_t)part_tokens / block_size + 2;
  return 1024 + ring + 2 * (size_t)stages * sizeof(uint64_t) + nbt * sizeof(int);
}

// (head_dim, compute warps, stages, n-tiles, FP8 caches).  Rings: bf16 64,
// 96 and 192 KB for head_dim 64, 128 and 256; FP8 64 KB (head_dim 64, 128:
// three CTAs per SM fit at 128) and 96 KB (256: two CTAs per SM; 128 with
// six stages, for one-wave grids of single-tile units).
#define PA_MMA_DISPATCH(CALL)                                                       \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 3 && k.n8 == 1 && !k.kv_fp8) \
    CALL(128, 4, 3, 1, false);                                                      \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 3 && k.n8 == 2 && !k.kv_fp8) \
    CALL(128, 4, 3, 2, false);                                                      \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 4 && k.n8 == 1 && !k.kv_fp8)  \
    CALL(64, 4, 4, 1, false);                                                       \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 4 && k.n8 == 2 && !k.kv_fp8)  \
    CALL(64, 4, 4, 2, false);                                                       \
  if (k.head_dim == 256 && k.consumer_warps == 4 && k.stages == 3 && k.n8 == 1 && !k.kv_fp8) \
    CALL(256, 4, 3, 1, false);                                                      \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 4 && k.n8 == 1 && k.kv_fp8)  \
    CALL(128, 4, 4, 1, true);                                                       \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 4 && k.n8 == 2 && k.kv_fp8)  \
    CALL(128, 4, 4, 2, true);                                                       \
  if (k.head_dim == 128 && k.consumer_warps == 4 && k.stages == 6 && k.n8 == 1 && k.kv_fp8)  \
    CALL(128, 4, 6, 1, true);                                                       \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 8 && k.n8 == 1 && k.kv_fp8)   \
    CALL(64, 4, 8, 1, true);                                                        \
  if (k.head_dim == 64 && k.consumer_warps == 4 && k.stages == 8 && k.n8 == 2 && k.kv_fp8)   \
    CALL(64, 4, 8, 2, true);                                                        \
  if (k.head_dim == 256 && k.consumer_warps == 4 && k.stages == 3 && k.n8 == 1 && k.kv_fp8)  \
    CALL(256, 4, 3, 1, true);

cudaError_t launch_partition_mma(const DecodeArgs& a, const KernelShape& k, const CUtensorMap& tk,
                                 const CUtensorMap& tv, dim3 grid, size_t smem,
                                 cudaStream_t stream) {
#define PA_CALL(D, N, S, N8, F8) return launch_mma_t<D, N, S, N8, F8>(a, tk, tv, grid, smem, stream)
  PA_MMA_DISPATCH(PA_CALL)
#undef PA_CALL
  return cudaErrorInvalidValue;
}

int occupancy_partition_mma(const KernelShape& k, size_t smem) {
#define PA_CALL(D, N, S, N8, F8) return occupancy_mma_t<D, N, S, N8, F8>(smem)
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

template <int D, int DSPLIT>
cudaError_t launch_reduce_t(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int PPW = 32 / (D / DSPLIT / 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_rows * DSPLIT, a.num_kv_heads, a.batch);
  // Warps per CTA, 1 to 32.  Few CTAs (one partition grid's worth of units
  // is small): latency decides, so each lane takes at most two partials and
  // all of them are in flight at once.  Many CTAs (the large-block MTP
  // workload: 16K of them, 16 partials each): they hide each other's
  // latency, so eight partials per lane (four rounds) keep the grid small.
  const long long ctas = (long long)cfg.gridDim.x * cfg.gridDim.y * cfg.gridDim.z;
  const int per_lane = ctas <= 1024 ? 2 : 8;
  const int nw = max(1, min(32, (a.max_parts + per_lane * PPW - 1) / (per_lane * PPW)));
  cfg.blockDim = dim3(32 * nw);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = pa_reduce_kernel<D, DSPLIT>;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// head_dim split of the reduce: the smallest of 1, 2, 4, ... (the first that
// gives a partial's slice <= 32 lanes) at which 16 warps, two partials per
// lane, cover the partials (only rows with more than 32 partials split):
// more, smaller CTAs pull a long row's partials from L2 in parallel and fold
// a shorter tree; far smaller ones (a lane per partial) load each partial's
// lse once per lane and lost again.
template <int D>
cudaError_t launch_reduce_d(const DecodeArgs& a, cudaStream_t stream) {
  auto fits = [&](int dsplit) { return 2 * 16 * (32 / (D / dsplit / 4)) >= a.max_parts; };
  if constexpr (D <= 128)
    if (fits(1)) return launch_reduce_t<D, 1>(a, stream);
  if (fits(2)) return launch_reduce_t<D, 2>(a, stream);
  if (fits(4)) return launch_reduce_t<D, 4>(a, stream);
  if (fits(8)) return launch_reduce_t<D, 8>(a, stream);
  return launch_reduce_t<D, 16>(a, stream);  // beyond this, lanes take more rounds
}

cudaError_t launch_reduce(const DecodeArgs& a, cudaStream_t stream) {
  if (a.head_dim == 128) return launch_reduce_d<128>(a, stream);
  if (a.head_dim == 64) return launch_reduce_d<64>(a, stream);
  if (a.head_dim == 256) return launch_reduce_d<256>(a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_ranges(int32_t* lo, int32_t* hi, const int32_t* seq_lens,
                          const int32_t* query_lens, int window, const int32_t* windows,
                          int batch, cudaStream_t stream) {
  pa_ranges_kernel<<<1, 1024, 0, stream>>>(lo, hi, seq_lens, query_lens, window, windows, batch);
  return cudaGetLastError();
}

cudaError_t launch_unreachable(int32_t* count, const int32_t* seq_lens, const int32_t* query_lens,
                               int window, const int32_t* windows, int block_shift, int batch,
                               cudaStream_t stream) {
  pa_unreachable_kernel<<<(batch + 255) / 256, 256, 0, stream>>>(count, seq_lens, query_lens, window,
                                                                  windows, block_shift, batch);
  return cudaGetLastError();
}

cudaError_t launch_stage(const StageArgs& s, cudaStream_t stream) {
  if (s.n <= 0 || s.n > kMaxStageCopies || s.blocks <= 0) return cudaErrorInvalidValue;
  pa_stage_kernel<<<s.blocks, 256, 0, stream>>>(s);
  return cudaGetLastError();
}

unsigned long long context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
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
