// pa_tc.cuh -- the tensor-memory partition kernel (tcgen05) for FP8 e4m3 KV
// caches with head_dim 128.  Included by pa_kernels.cu inside its anonymous
// namespace (it uses the status word and the helpers defined there).
//
// Same partition, same partials as the other partition kernels: split-K
// flash-decoding (ExecuTorch PR #18759) over a paged cache (gllm PR #116).
// The difference is where the arithmetic runs.  The mma.sync path converts
// every FP8 code to f16 in registers before it can use it; here the codes go
// from the TMA-filled shared-memory ring straight into tcgen05.mma
// (kind::f8f6f4, e4m3 x e4m3 -> fp32 in tensor memory):
//
//   S^T[128 tokens x 16 rows]  = K[128 x 128 d]  . Q^T[128 d x 16 rows]
//   O_w[128 d x 16 rows]       = V_w^T[128 d x 32 tokens] . P_w^T[32 tokens x 16 rows]
//
// with the KV tokens on the MMA's M axis (M = 128) and the unit's query rows
// padded to N = 16.  A stage is 128 tokens.  Q and P enter as e4m3 too: a bf16
// q row is scaled by a power of two sig that puts its largest |q| in
// [128, 256) and split into hi + lo e4m3 terms (hi carries the top four
// significant bits, lo the next four: exact for every element within 2^9 of
// the row's largest); an FP8 q is one term.  P (in [0, 1]) is scaled by 256
// and split the same way.  Each split doubles the MMAs of its product, which
// the tensor cores have to spare on this HBM-bound path.
//
// Roles (320 threads): warp 0 copies (TMA ring), warp 1 issues the MMAs from
// one thread and owns the tensor-memory allocation, warps 2..9 (256 threads)
// run the softmax and accumulate O.  Warp w may only touch TMEM lanes
// 32*(w%4)..+31, so softmax warp w owns tokens 32*(w%4)..+31 of each stage
// (as rows of S^T) and dims 32*(w%4)..+31 (as rows of O), for half of the
// query rows (two warps per lane quadrant, so twice the warps hide the
// softmax's dependent chain).  Each softmax warp keeps its own running max
// per row over its 32-token slice of every
// stage, so no statistic crosses warps until the partition ends; the PV
// product is therefore issued per slice (four K = 32 MMAs into four O
// buffers), and each thread folds the four per-stage O slices into registers
// with their slices' rescale factors.
//
// Pipeline, per stage k: copy warp fills ring slot k % NS; MMA thread issues
// S(k) into TMEM buffer k % 2 (commit -> s_full), then PV(k-1) once P(k-1)
// is written and O(k-2) has been read (commit -> o_full, and -> the ring
// slot's empty barrier); softmax warps read S(k) (-> s_free), write P(k) and
// the slice rescale factors (-> p_full), then read O(k-1) (-> o_free).  Every
// wait is bounded; on a timeout the status word records it and every role
// still reaches the teardown, where the allocating warp waits for the MMAs
// in flight before it frees the tensor memory.
// ---------------------------------------------------------------------------

constexpr int kTcStage = 128;     // tokens per stage
constexpr int kTcN = 16;          // MMA N: query rows per CTA, padded
constexpr int kTcTmemCols = 128;  // S: 2 x 16 columns, O: 4 x 16 columns (96 used)

struct TcLayout {
  static constexpr int ROW = 128;                    // bytes per FP8 token row (head_dim 128)
  static constexpr int KV_BYTES = kTcStage * ROW;    // 16 KB
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;   // K then V
  static constexpr int QB_BYTES = kTcN * ROW;        // one Q^T term: 16 rows x 128 B
  static constexpr int PB_BYTES = kTcN * kTcStage;   // one P^T term: 16 rows x 128 tokens
};

// ---- tcgen05 wrappers -------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start
// address, leading and stride byte offsets in 16-byte units, version 1,
// layout type 2 = SWIZZLE_128B).
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f8f6f4, e4m3 x e4m3 -> fp32, M x N.
__host__ __device__ constexpr uint32_t tc_idesc(int m, int n, int a_mn_major, int b_mn_major) {
  return (1u << 4)                                         // D format: fp32
         | (0u << 7) | (0u << 10)                          // A, B: e4m3
         | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16)
         | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every tcgen05 operation this thread issued has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar)
               : "memory");
}

template <int NC>
__device__ __forceinline__ void tc_ld(uint32_t taddr, float (&v)[NC]) {
  static_assert(NC == 4 || NC == 8 || NC == 16, "4, 8 or 16 columns");
  uint32_t r[NC];
  if constexpr (NC == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (NC == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
#pragma unroll
  for (int i = 0; i < NC; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Byte offset of byte `col` (0..127) of row r in a 16-row, 128-byte-row tile
// laid out for the 128-byte swizzle (rows in 1024-byte groups of 8).
__device__ __forceinline__ uint32_t tc_sw128(int r, int col) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((col >> 4) ^ (r & 7))) << 4) + (col & 15));
}

// Max over the 32 lanes of v[r] for every r < RT, result in every lane: one
// redux.sync per row on an integer key that orders like the float (sign-
// magnitude flipped for negatives; -inf maps to a valid key).
__device__ __forceinline__ int tc_fkey(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7fffffff);
}
__device__ __forceinline__ float tc_unkey(int k) {
  return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff));
}

template <int RT>
__device__ __forceinline__ void tc_warp_rowmax(const float (&v)[RT], float (&out)[RT]) {
#pragma unroll
  for (int r = 0; r < RT; ++r) out[r] = tc_unkey(__reduce_max_sync(FULL, tc_fkey(v[r])));
}

// At 80 registers six warps share an SM sub-partition's register file, so
// two 10-warp CTAs fit an SM however their warps are spread.
template <int NS, int RT>
__global__ void __maxnreg__(80)
    pa_partition_tc_kernel(const __grid_constant__ DecodeArgs a,
                           const __grid_constant__ CUtensorMap tmk,
                           const __grid_constant__ CUtensorMap tmv) {
  constexpr int D = 128;
  using Lt = TcLayout;
  static_assert(RT == 8 || RT == 16, "rows per CTA");
  constexpr int NSW = 8;       // softmax warps: two per TMEM lane quadrant
  constexpr int RW = RT / 2;   // rows per softmax warp

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* qsm = smem + NS * Lt::STAGE_BYTES;  // [2 terms][16 rows][128 B], swizzled
  uint8_t* psm = qsm + 2 * Lt::QB_BYTES;       // [2 buffers][2 terms][16 rows][128 tokens]
  uint64_t* bars = reinterpret_cast<uint64_t*>(psm + 4 * Lt::PB_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* s_full = bars + 2 * NS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_free = o_full + 1;
  uint64_t* mma_done = o_free + 1;
  float* alpha_s = reinterpret_cast<float*>(mma_done + 1);  // [2 buffers][4 slices][16 rows]
  float* stat_m = alpha_s + 2 * 4 * kTcN;                    // [4 slices][16 rows]
  float* stat_l = stat_m + 4 * kTcN;
  float* sig_s = stat_l + 4 * kTcN;                          // [16 rows]
  int* bt_s = reinterpret_cast<int*>(sig_s + kTcN);

  __shared__ uint32_t s_tmem;
  __shared__ int s_c0[NS];
  __shared__ int s_lo[kTcN], s_hi[kTcN];  // visible range of each row (empty for padding rows)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  const int kvh = blockIdx.y % a.num_kv_heads;
  const int slab = blockIdx.y / a.num_kv_heads;
  const int part = blockIdx.x;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full[s]), 1);   // copy-warp arrival + tx bytes
      mbar_init(smem_u32(&empty[s]), 1);  // the MMA thread's commit after PV
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), NSW);
      mbar_init(smem_u32(&p_full[i]), NSW);
    }
    mbar_init(smem_u32(o_full), 1);
    mbar_init(smem_u32(o_free), NSW);
    mbar_init(smem_u32(mma_done), 1);
    fence_mbar_init();
  }
  __syncthreads();  // barriers initialised for every role
  asm volatile("griddepcontrol.wait;" ::: "memory");

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
  const int A = ulo & ~(kStageTokens - 1);
  const int nparts = (S - A + a.part_tokens - 1) / a.part_tokens;
  if (R > a.max_rows || nparts > a.max_parts) {
    if (lead) atomicOr(&g_pa_status, PA_DEV_HINT);
    return;
  }
  const int row0 = slab * a.slab_rows;
  if (row0 >= R || part >= nparts) return;
  const int Rs = min(RT, R - row0);
  const int p0 = A + part * a.part_tokens;
  const int p1 = min(S, p0 + a.part_tokens);
  const int nst = (p1 - p0 + kTcStage - 1) / kTcStage;
  const int jb0 = p0 >> a.block_shift;
  const int nbt = ((p1 - 1) >> a.block_shift) - jb0 + 1;
  const int qoff = row_token_offset(a.query_lens, b, lane);

  // ---- set-up: tensor memory, Q^T terms, zeroed P buffers ----------------
  // (the copy warp skips it and starts on the block table at once)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTcTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp >= 2 && warp < 6) {
    const int t = threadIdx.x - 64;  // 0..127: (row t/8, 16-dim chunk t%8)
    const int r = t >> 3, c = t & 7;
    uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = make_uint4(0u, 0u, 0u, 0u);
    size_t qrow = 0;
    const bool has = r < Rs;
    if (has) {
      const int rr = row0 + r;
      const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
      qrow = ((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D;
    }
    float sig = 1.f;
    if (a.q_fp8) {
      if (has) hi = __ldg(reinterpret_cast<const uint4*>(a.q8 + qrow) + c);
    } else {
      uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
      if (has) {
        w0 = __ldg(reinterpret_cast<const uint4*>(a.q + qrow) + 2 * c);
        w1 = __ldg(reinterpret_cast<const uint4*>(a.q + qrow) + 2 * c + 1);
      }
      float x[16];
      const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float2 f = bf2_to_f2(wv[u]);
        x[2 * u] = f.x;
        x[2 * u + 1] = f.y;
      }
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) amax = fmaxf(amax, fabsf(x[u]));
      amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 4));
      // amax in [2^E, 2^(E+1)) -> sig = 2^(E-7); rows below 2^-119 keep sig = 1
      const int ebits = (__float_as_int(amax) >> 23) & 0xff;
      sig = ebits >= 8 ? __int_as_float((ebits - 7) << 23) : 1.f;
      const float isig = ebits >= 8 ? __int_as_float((261 - ebits) << 23) : 1.f;
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x0 = x[4 * u] * isig, x1 = x[4 * u + 1] * isig;
        const float x2 = x[4 * u + 2] * isig, x3 = x[4 * u + 3] * isig;
        const uint32_t h01 = f32x2_to_e4m3x2(x0, x1), h23 = f32x2_to_e4m3x2(x2, x3);
        const uint32_t hf01 = e4m3x2_to_f16x2(h01), hf23 = e4m3x2_to_f16x2(h23);
        const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&hf01));
        const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&hf23));
        hw[u] = h01 | (h23 << 16);
        lw[u] = f32x2_to_e4m3x2(x0 - g01.x, x1 - g01.y) |
                (f32x2_to_e4m3x2(x2 - g23.x, x3 - g23.y) << 16);
      }
      hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    const uint32_t off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
    *reinterpret_cast<uint4*>(qsm + off) = hi;
    *reinterpret_cast<uint4*>(qsm + Lt::QB_BYTES + off) = lo;
    if (c == 0) {
      sig_s[r] = sig;
      int lo = INT_MAX, hi = INT_MIN;
      if (has) query_range(S, L, (row0 + r) / a.group, w, lo, hi);
      s_lo[r] = lo;
      s_hi[r] = hi;
    }
    fence_proxy_async_smem();  // the tensor core reads Q through the async proxy
  }
  if (warp >= 2) {
    // P buffers start at zero: rows >= Rs are never written again
    const int t = threadIdx.x - 64;  // 0..255
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 2; ++u)
      *reinterpret_cast<uint4*>(psm + (size_t)(u * 256 + t) * 16) = z;
    fence_proxy_async_smem();
  }
  uint32_t tmem = 0;
  if (warp != 0) {
    tc_fence_before();
    named_bar_sync(2, 32 + 32 * NSW);  // MMA and softmax warps: tensor memory, Q and P ready
    tc_fence_after();
    tmem = s_tmem;
  }

  const int BR = min(a.block_size, kStageTokens);
  const uint32_t box_bytes = (uint32_t)BR * Lt::ROW;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------ copy warp ------------------------------
    for (int i = lane; i < nbt; i += 32) {
      int phys = a.block_tables[(size_t)b * a.max_blocks_per_seq + jb0 + i];
      if (phys < 0 || phys >= a.num_blocks) {
        atomicOr(&g_pa_status, PA_DEV_BAD_BLOCK);
        phys = -1;
      }
      bt_s[i] = phys;
    }
    __syncwarp();
    const int nbox = kTcStage / BR;
    const int nitem = nbox * 2;  // (box, K/V) per lane: at most 16
    const uint64_t kv_policy = l2_evict_first_policy();  // K/V codes are read once
    int k = 0;
    for (; k < nst; ++k) {
      const int s = k % NS;
      if (k >= NS) {
        bool got = true;
        if (lane == 0) got = mbar_wait(smem_u32(&empty[s]), ((k / NS) - 1) & 1);
        if (!__shfl_sync(FULL, got, 0)) {
          ok = false;
          break;
        }
      }
      const int c0 = p0 + k * kTcStage;
      const int ta = max(c0, ulo), te = min(c0 + kTcStage, p1);
      bool mine = false;
      uint32_t dst = 0;
      int y = 0, isv = 0;
      if (lane < nitem) {
        const int j = lane >> 1;
        isv = lane & 1;
        const int bt0 = c0 + j * BR;
        if (bt0 + BR > ta && bt0 < te) {
          const int jj = bt0 >> a.block_shift;
          const int phys = bt_s[jj - jb0];
          if (phys >= 0) {
            mine = true;
            y = (phys * a.num_kv_heads + kvh) * a.block_size + (bt0 - (jj << a.block_shift));
            dst = s * Lt::STAGE_BYTES + isv * Lt::KV_BYTES + j * box_bytes;
          }
        }
      }
      const uint32_t nload = __popc(__ballot_sync(FULL, mine));
      if (lane == 0) {
        s_c0[s] = c0;
        mbar_arrive_expect_tx(smem_u32(&full[s]), nload * box_bytes);
      }
      __syncwarp();
      if (mine)
        tma_load_3d_hint(smem_u32(smem) + dst,
                         isv ? static_cast<const void*>(&tmv) : static_cast<const void*>(&tmk), 0,
                         y, 0, smem_u32(&full[s]), kv_policy);
    }
    const int issued = k;
    if (ok && lane == 0) {
      // the stop stage: its slot last held stage issued - NS
      const int s = issued % NS;
      bool got = true;
      if (issued >= NS) got = mbar_wait(smem_u32(&empty[s]), ((issued / NS) - 1) & 1);
      if (got) {
        s_c0[s] = -1;
        mbar_arrive(smem_u32(&full[s]));
      }
    }
    if (lane == 0) {
      for (int kk = max(0, issued - NS + 1); kk < issued; ++kk)
        mbar_wait(smem_u32(&full[kk % NS]), (kk / NS) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------- MMA thread ----------------------------
    if (lane == 0) {
      constexpr uint32_t kIdescQK = tc_idesc(128, kTcN, 0, 0);  // K . Q^T: both K-major
      constexpr uint32_t kIdescPV = tc_idesc(128, kTcN, 1, 0);  // V^T (d-contiguous) . P^T
      const bool two = !a.q_fp8;
      const uint32_t qa = smem_u32(qsm), pa = smem_u32(psm);
      for (int k = 0;; ++k) {
        const int s = k % NS;
        bool stop = true;
        if (mbar_wait(smem_u32(&full[s]), (k / NS) & 1)) stop = s_c0[s] < 0;
        if (!stop && k >= 2 && !mbar_wait(smem_u32(&s_free[k & 1]), ((k - 2) >> 1) & 1))
          stop = true;
        if (!stop) {
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + s * Lt::STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t ad = tc_desc(ka + 32 * kk, 16, 1024);
            tc_mma(tmem + (k & 1) * kTcN, ad, tc_desc(qa + 32 * kk, 16, 1024), kIdescQK, kk > 0);
            if (two)
              tc_mma(tmem + (k & 1) * kTcN, ad, tc_desc(qa + Lt::QB_BYTES + 32 * kk, 16, 1024),
                     kIdescQK, 1);
          }
          tc_commit(smem_u32(&s_full[k & 1]));
        }
        if (k >= 1) {
          // PV of the previous stage
          const int pk = k - 1, ps = pk % NS;
          bool go = mbar_wait(smem_u32(&p_full[pk & 1]), (pk >> 1) & 1);
          if (go && pk >= 1) go = mbar_wait(smem_u32(o_free), (pk - 1) & 1);
          if (go) {
            tc_fence_after();
            const uint32_t va = smem_u32(smem + ps * Lt::STAGE_BYTES + Lt::KV_BYTES);
            const uint32_t pb = pa + (pk & 1) * 2 * Lt::PB_BYTES;
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
              const uint64_t ad = tc_desc(va + sl * 32 * Lt::ROW, 0, 1024);
              tc_mma(tmem + 2 * kTcN + sl * kTcN, ad, tc_desc(pb + 32 * sl, 16, 1024), kIdescPV,
                     0);
              tc_mma(tmem + 2 * kTcN + sl * kTcN, ad,
                     tc_desc(pb + Lt::PB_BYTES + 32 * sl, 16, 1024), kIdescPV, 1);
            }
            tc_commit(smem_u32(o_full));
            tc_commit(smem_u32(&empty[ps]));
          } else {
            stop = true;
          }
        }
        if (stop) break;
      }
      tc_commit(smem_u32(mma_done));
    }
    __syncwarp();
  } else {
    // ---------------------------- softmax warps ----------------------------
    const int qd = warp & 3;               // TMEM lane quadrant of this warp
    const int r0w = ((warp - 2) >> 2) * RW;  // first of this warp's rows
    const int tk = 32 * qd + lane;         // my token within a stage; my dim of O
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    // (per-row scale and range live in smem: broadcast reads, no registers)
    float m_w[RW], l_p[RW], acc[4][RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      m_w[r] = kNegInf;
      l_p[r] = 0.f;
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) acc[sl][r] = 0.f;
    }
    for (int k = 0;; ++k) {
      named_bar_sync(1, 32 * NSW);  // the softmax warps move in step
      const int s = k % NS;
      // (every decision below is warp-uniform: the tcgen05 loads are .sync.aligned)
      int c0 = -1;
      if (ok) {
        if (__all_sync(FULL, mbar_wait(smem_u32(&full[s]), (k / NS) & 1)))
          c0 = s_c0[s];
        else
          ok = false;
      }
      if (c0 >= 0 && !__all_sync(FULL, mbar_wait(smem_u32(&s_full[k & 1]), (k >> 1) & 1))) {
        ok = false;
        c0 = -1;
      }
      if (c0 >= 0) {
        tc_fence_after();
        float sv[RW];
        tc_ld<RW>(tl + (k & 1) * kTcN + r0w, sv);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s_free[k & 1]));
        const int t = c0 + tk;
        float v[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r)
          v[r] = (t >= s_lo[r0w + r] && t < s_hi[r0w + r])
                     ? sv[r] * (a.scale_log2 * sig_s[r0w + r])
                     : kNegInf;
        float wm[RW];
        tc_warp_rowmax<RW>(v, wm);
        float al[RW], p[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          const float mn = fmaxf(m_w[r], wm[r]);
          const float mu = (mn == kNegInf) ? 0.f : mn;
          al[r] = (mn == kNegInf) ? 1.f : ex2(m_w[r] - mu);
          m_w[r] = mn;
          p[r] = ex2(v[r] - mu);
          l_p[r] = l_p[r] * al[r] + p[r];
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
          if (lane == r) alpha_s[(k & 1) * 4 * kTcN + qd * kTcN + r0w + r] = al[r];
        // P^T (x 256) as hi + lo e4m3 terms, one byte per (row, token)
        uint8_t* pb = psm + (k & 1) * 2 * Lt::PB_BYTES;
#pragma unroll
        for (int r = 0; r < RW; r += 2) {
          const float x0 = p[r] * 256.f, x1 = p[r + 1] * 256.f;
          const uint32_t h = f32x2_to_e4m3x2(x0, x1);
          const uint32_t hf = e4m3x2_to_f16x2(h);
          const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&hf));
          const uint32_t lw = f32x2_to_e4m3x2(x0 - g.x, x1 - g.y);
          const uint32_t o0 = tc_sw128(r0w + r, tk), o1 = tc_sw128(r0w + r + 1, tk);
          pb[o0] = (uint8_t)(h & 0xffu);
          pb[o1] = (uint8_t)(h >> 8);
          pb[Lt::PB_BYTES + o0] = (uint8_t)(lw & 0xffu);
          pb[Lt::PB_BYTES + o1] = (uint8_t)(lw >> 8);
        }
        // V rows of tokens outside the row's union span may hold anything
        // (uninitialised cache slots, earlier stages): zero them so the PV
        // product never multiplies a 0 weight by a NaN.  The two warps of a
        // quadrant zero one half of the row each.
        if (t < ulo || t >= p1) {
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          uint4* vr = reinterpret_cast<uint4*>(smem + s * Lt::STAGE_BYTES + Lt::KV_BYTES +
                                               tk * Lt::ROW) +
                      (r0w ? 4 : 0);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) vr[cc] = z;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[k & 1]));
      }
      if (k >= 1) {
        // fold O of the previous stage into registers (thread = dim tk)
        const int pk = k - 1;
        const bool got = ok && __all_sync(FULL, mbar_wait(smem_u32(o_full), pk & 1));
        if (got) {
          tc_fence_after();
          float ov[4][RW];
#pragma unroll
          for (int sl = 0; sl < 4; ++sl) tc_ld<RW>(tl + 2 * kTcN + sl * kTcN + r0w, ov[sl]);
          tc_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(o_free));
          const float* alp = alpha_s + (pk & 1) * 4 * kTcN + r0w;
#pragma unroll
          for (int sl = 0; sl < 4; ++sl)
#pragma unroll
            for (int r = 0; r < RW; ++r) acc[sl][r] = acc[sl][r] * alp[sl * kTcN + r] + ov[sl][r];
        } else {
          ok = false;
        }
      }
      if (c0 < 0) break;
    }

    // ---- merge the four token slices and write the partial --------------
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      float ls = l_p[r];
#pragma unroll
      for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(FULL, ls, o);
      if (lane == r) {
        stat_m[qd * kTcN + r0w + r] = m_w[r];
        stat_l[qd * kTcN + r0w + r] = ls;
      }
    }
    named_bar_sync(1, 32 * NSW);
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int row = r0w + r;
      if (row >= Rs) continue;
      float M = kNegInf;
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) M = fmaxf(M, stat_m[sl * kTcN + row]);
      float Z = 0.f, O = 0.f;
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        const float f = (M == kNegInf) ? 0.f : ex2(stat_m[sl * kTcN + row] - M);
        Z += f * stat_l[sl * kTcN + row];
        O += f * acc[sl][r];
      }
      const int rr = row0 + row;
      const float inv = Z > 0.f ? a.v_scale / (256.f * Z) : 0.f;
      if (nparts == 1) {
        const int i = rr / a.group, j = rr - (rr / a.group) * a.group;
        a.dst[((size_t)(qoff + i) * a.num_q_heads + (size_t)kvh * a.group + j) * D + tk] =
            __float2bfloat16_rn(O * inv);
      } else {
        const size_t base =
            ((size_t)(b * a.num_kv_heads + kvh) * a.max_parts + part) * a.max_rows + rr;
        a.ws_o[base * D + tk] = O * inv;
        if (tk == 0) a.ws_lse[base] = Z > 0.f ? M + lg2(Z) : kNegInf;
      }
    }
  }

  // ---- teardown: wait for the MMAs in flight, then free tensor memory ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(smem_u32(mma_done), 0);
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcTmemCols));
  }
}
