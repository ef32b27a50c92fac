// Block-sparse flash attention of Sparse VideoGen (arXiv 2502.01776 abstract:
// "customized kernel implementations" for the spatial/temporal sparse 3D
// attention; the project article "Sparse-VideoGen and the sparsity hiding
// inside video diffusion attention" names block sparse attention with varied
// block sizes). For every query block the kernel walks that block's CSR list of
// key blocks; every listed (query block, key block) pair is attended in full.
//
// One CTA = one (b*H + h, query block). 192 threads, warp-specialised:
//   warps 0-3  softmax + epilogue; thread t owns query row t = TMEM lane t
//   warp 4     TMA producer: the Q tile once, then K/V tiles of the listed
//              key blocks into a ring of shared-memory stages
//   warp 5     MMA issuer (one thread): S = Q K^T (both operands in shared
//              memory, 128-byte swizzle) and O += P V (P from tensor memory,
//              V from shared memory) with tcgen05.mma, fp32 accumulators in
//              tensor memory
// Tensor memory (512 columns): S double buffer at columns 0 and 128, O at 256.
// P (bf16) overwrites the first half of its S buffer. While the softmax warps
// work on S_j the tensor core already computes S_{j+1}; P_j V_j follows as
// soon as P_j is written. The running maximum is re-based lazily (only when
// a tile's maximum exceeds it by more than 2^8), so O is rarely rescaled.
// All barrier waits are bounded (see sm100.cuh).
#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr float kRebaseLog2 = 8.0f;  // lazy re-basing threshold (log2 units)

struct Barriers {
  uint64_t q_full;
  uint64_t k_full[3], v_full[3], kv_empty[3];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full, o_final, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int BK>
struct Cfg {
  static constexpr int kPanels = D / 64;            // 128-byte wide column panels
  static constexpr int kQPanel = 128 * 128;         // 128 rows x 128 B
  static constexpr int kKVPanel = BK * 128;         // BK rows x 128 B
  static constexpr int kQBytes = kPanels * kQPanel;
  static constexpr int kKVBytes = kPanels * kKVPanel;  // one K (or V) tile
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(Barriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;  // + alignment slack
  // Keep one CTA per SM: each CTA takes all 512 tensor-memory columns.
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static_assert(kOffBar + kBarBytes + 1024 <= kSmem, "bookkeeping must fit the allocation");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

// Tensor maps [1] are the position-major copies (3-D tiled maps), or, with
// `gather` set, a 2-D row map (box 64 x 1) over the frame-major q from which
// temporal heads gather their query rows in position-major order; k and v
// likewise with `gather_kv`, else tiled maps over position-major copies.
struct __align__(64) AttnParams {
  CUtensorMap tm_q[2], tm_k[2], tm_v[2];  // [0]: frame-major, [1]: position-major
  // FP8 PV: e4m3 V of every head in its own layout (one 8-bit tiled map) and
  // the per-(head, channel) scales that undo its quantisation
  CUtensorMap tm_v8;
  const float* v_scale;
  const int8_t* labels;
  const int32_t* row_ptr[2];
  const int32_t* col_idx[2];
  svg_bf16* out[2];
  float* lse;
  int* status;
  int32_t N, Nv, BH, nqb, nkb, bq, bk;
  int32_t has_permuted;
  int32_t csr_per_head;  // CSR row of (bh, query block r) is bh * nqb + r
  int32_t gather, gather_kv, T, P;
  float scale_log2;
};


__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// Frame-major row of position-major row j (the inverse of the layout
// transformation pi(f*P + p) = p*T + f; text rows stay in place). Rows past
// the end are clamped to the last row: they only fill the ragged tail of a
// tile, whose keys the softmax masks and whose query rows are never stored.
__device__ __forceinline__ int frame_major_row(int j, int N, int Nv, int T, int P) {
  if (j >= N) j = N - 1;
  if (j >= Nv) return j;
  const int pos = j / T;
  return (j - pos * T) * P + pos;
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attention_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  Barriers* bar = reinterpret_cast<Barriers*>(smem + C::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int qb = p.nqb - 1 - static_cast<int>(blockIdx.x);  // text-heavy (longest) rows first
  const int bh = blockIdx.y;

  const int label = p.labels ? static_cast<int>(p.labels[bh]) : SVG_HEAD_SPATIAL;
  const int sel = label == SVG_HEAD_TEMPORAL ? 1 : 0;
  if (label != SVG_HEAD_SPATIAL && label != SVG_HEAD_TEMPORAL) {
    if (tid == 0) atomicOr(p.status, kDevErrBounds);
    return;
  }
  if (sel == 1 && !p.has_permuted) {
    if (tid == 0) atomicOr(p.status, kDevErrBounds);
    return;
  }
  const int csr_row = (p.csr_per_head ? bh * p.nqb : 0) + qb;
  const int32_t rp0 = __ldg(p.row_ptr[sel] + csr_row);
  int32_t n = __ldg(p.row_ptr[sel] + csr_row + 1) - rp0;
  if (n < 0 || n > p.nkb) {
    if (tid == 0) atomicOr(p.status, kDevErrBounds);
    n = 0;
  }
  const int32_t* cols = p.col_idx[sel] + rp0;

  // ---- set-up: barriers, tensor memory, padding rows of a short Q tile
  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 128);
    }
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_final, 1);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  if (p.bq < 128 && tid < 128 && tid >= p.bq) {
    for (int pn = 0; pn < C::kPanels; ++pn) {
      uint4* row = reinterpret_cast<uint4*>(sQ + pn * C::kQPanel + tid * 128);
#pragma unroll
      for (int i = 0; i < 8; ++i) row[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane_id() == 0 && n > 0) {
      const CUtensorMap* mq = &p.tm_q[sel];
      const CUtensorMap* mk = &p.tm_k[sel];
      const CUtensorMap* mv = &p.tm_v[sel];
      const uint64_t keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bar->q_full, static_cast<uint32_t>(p.bq * D * 2));
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_3d(sQ + pn * C::kQPanel, mq, &bar->q_full, pn * 64, qb * p.bq, bh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::kStages;
        if (!mbar_wait(&bar->kv_empty[st], ((j / C::kStages) & 1) ^ 1, abort_flag, p.status))
          break;
        int c = __ldg(cols + j);
        if (c < 0 || c >= p.nkb) c = 0;  // flagged and masked by the softmax warps
        mbar_arrive_expect_tx(&bar->k_full[st], C::kKVBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(sK + st * C::kKVBytes + pn * C::kKVPanel, mk, &bar->k_full[st],
                           pn * 64, c * BK, bh, keep);
        mbar_arrive_expect_tx(&bar->v_full[st], C::kKVBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(sV + st * C::kKVBytes + pn * C::kKVPanel, mv, &bar->v_full[st],
                           pn * 64, c * BK, bh, keep);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA retires.
        for (int j = (issued > C::kStages ? issued - C::kStages : 0); j < issued; ++j) {
          const int st = j % C::kStages;
          const uint32_t par = (j / C::kStages) & 1;
          int spare = 0;
          long long t0 = clock64();
          while (!(mbar_try_wait(&bar->k_full[st], par) && mbar_try_wait(&bar->v_full[st], par)) &&
                 clock64() - t0 < kWaitLimitCycles)
            ++spare;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane_id() == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BK, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      bool ok = mbar_wait(&bar->q_full, 0, abort_flag, p.status);
      tc_fence_after();
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % C::kStages;
          const uint32_t s_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->k_full[st], (j / C::kStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 16 bf16 of K inside the 128-byte row
            const uint64_t a = sdesc_sw128(q_addr + (kk >> 2) * C::kQPanel + off, 16, 1024);
            const uint64_t b =
                sdesc_sw128(k_addr + st * C::kKVBytes + (kk >> 2) * C::kKVPanel + off, 16, 1024);
            mma_bf16_ss(s_col, a, b, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full[j & 1]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % C::kStages;
          const uint32_t p_col = tmem + ((jj & 1) ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->p_full[jj & 1], (jj >> 1) & 1, abort_flag, p.status)) break;
          if (!mbar_wait(&bar->v_full[st], (jj / C::kStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t b = sdesc_sw128(v_addr + st * C::kKVBytes + kk * 16 * 128,
                                           C::kKVPanel, 1024);
            mma_bf16_ts(tmem + C::kColO, p_col + kk * 8, b, idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bar->kv_empty[st]);
          tc_commit(&bar->o_full);
          if (jj == n - 1) tc_commit(&bar->o_final);
        }
      }
      if (*abort_flag) {
        // Retire every MMA issued so far before tensor memory is released.
        tc_commit(&bar->drain);
        long long t0 = clock64();
        while (!mbar_try_wait(&bar->drain, 0) && clock64() - t0 < kWaitLimitCycles) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = qb * p.bq + tid;
    const bool row_valid = tid < p.bq && row < p.N;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY;  // running base, log2 units
    float l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t s_col = lane_base + (sb ? C::kColS1 : C::kColS0);
      const int c = __ldg(cols + j);
      const bool bad = c < 0 || c >= p.nkb;
      if (bad && tid == 0) atomicOr(p.status, kDevErrBounds);
      int kvalid = bad ? 0 : p.N - c * BK;
      if (kvalid > BK) kvalid = BK;
      if (!mbar_wait(&bar->s_full[sb], (j >> 1) & 1, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[BK];
#pragma unroll
      for (int ch = 0; ch < BK / 32; ++ch)
        tmem_ld_32x32b_x32(s_col + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      tmem_ld_wait();
      reg_fence(sr);

      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < BK; ++i) {
        const float x = i < kvalid ? u2f(sr[i]) : -INFINITY;
        mx = fmaxf(mx, x);
      }
      const float m_tile = mx * p.scale_log2;
      const bool rebase = m_tile > m + kRebaseLog2;
      const float m_new = rebase ? m_tile : m;
      const float alpha = rebase ? fast_exp2(m - m_new) : 1.0f;  // exp2(-inf) = 0
      const float m_use = m_new == -INFINITY ? 0.0f : m_new;

      float sum = 0.0f;
#pragma unroll
      for (int ch = 0; ch < BK / 32; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c0 = ch * 32 + 2 * i;
          const float p0 =
              c0 < kvalid ? fast_exp2(fmaf(u2f(sr[c0]), p.scale_log2, -m_use)) : 0.0f;
          const float p1 =
              c0 + 1 < kvalid ? fast_exp2(fmaf(u2f(sr[c0 + 1]), p.scale_log2, -m_use)) : 0.0f;
          sum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st_32x32b_x16(s_col + ch * 16, pk);
      }
      l = l * alpha + sum;
      m = m_new;
      tmem_st_wait();

      // Re-base O (PV_{j-1} must have landed) when any row of this warp moved.
      if (j > 0 && __any_sync(0xffffffffu, rebase)) {
        if (!mbar_wait(&bar->o_full, (j - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(lane_base + C::kColO + ch * 32, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * alpha);
          tmem_st_32x32b_x32(lane_base + C::kColO + ch * 32, o);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[sb]);
    }

    // ---- epilogue: O / l -> bf16, lse
    if (ok && n > 0) ok = mbar_wait(&bar->o_final, 0, abort_flag, p.status);
    tc_fence_after();
    svg_bf16* out = p.out[sel] + (static_cast<size_t>(bh) * p.N + row) * D;
    const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
    const bool have_o = ok && n > 0;
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld_32x32b_x32(lane_base + C::kColO + ch * 32, o);
        tmem_ld_wait();
        reg_fence(o);
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = have_o ? pack_bf16x2(u2f(o[2 * i]) * inv_l, u2f(o[2 * i + 1]) * inv_l) : 0u;
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + ch * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
    }
    if (p.lse != nullptr && row_valid) {
      p.lse[static_cast<size_t>(bh) * p.N + row] =
          (have_o && l > 0.0f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ===========================================================================
// Paired-tile variant (block_q = 128): one CTA = two consecutive query blocks
// A = 2p and B = 2p+1 of one head. The K/V tiles of the union of the two CSR
// rows stream once through separate K and V rings and serve both tiles.
// 384 threads (three warpgroups): warps 0-3 softmax of tile A, warps 4-7
// softmax of tile B, warp 8 TMA producer, warp 9 MMA issuer, warps 10-11 idle.
// The kernel launches at 168 registers per thread (three warps per SM
// sub-partition); the producer warpgroup then gives registers back
// (setmaxnreg.dec to 56) and the softmax warpgroups take them (setmaxnreg.inc
// to 224): 224 + 224 + 56 = 3 x 168 per sub-partition. Tensor memory: S_A 0, O_A 128,
// S_B 256, O_B 384 (P_t overwrites the first half of S_t). Per union step u
// the MMA issue order is PV_A(u-1), QK_A(u), PV_B(u-1), QK_B(u): each tile's
// softmax overlaps the other tile's PV and QK, every PV is issued at most one
// step after its block, and PV_t(j-1) always precedes QK_t(j), so the commit of
// S_t(j) also retires PV_t(j-1) (the softmax may then re-base O_t freely).
// ===========================================================================
constexpr int kPairThreads = 384;
constexpr float kRebaseLog2F8 = 2.0f;  // FP8 PV: lazy re-basing threshold (log2 units)
constexpr float kPShiftLog2F8 = 6.0f;  // FP8 PV: P is scaled by 2^6 before rounding
constexpr int kPairProducerWarp = 8;
constexpr int kPairMmaWarp = 9;
constexpr int kPairLaunchRegs = 168;   // per thread at launch (3 warps per sub-partition)
constexpr int kPairSoftmaxRegs = 224;  // softmax warpgroups after setmaxnreg.inc
constexpr int kPairOtherRegs = 56;     // producer / MMA warpgroup after setmaxnreg.dec
static_assert(2 * kPairSoftmaxRegs + kPairOtherRegs == 3 * kPairLaunchRegs,
              "register split must equal the launch allocation");

struct PairBarriers {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int BK, bool F8 = false>
struct PairCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kQPanel = 128 * 128;
  static constexpr int kKVPanel = BK * 128;
  static constexpr int kQBytes = kPanels * kQPanel;     // one query tile
  static constexpr int kKVBytes = kPanels * kKVPanel;   // one K (or bf16 V) tile
  // FP8 PV: a V tile is BK rows of D = 128 e4m3 bytes, one 128-byte swizzled panel
  static constexpr int kVBytes = F8 ? BK * 128 : kKVBytes;
  static constexpr int kKStages = (D == 128 && BK == 128) ? 2 : 3;
  static constexpr int kVStages = F8 ? 3 : kKStages;
  static constexpr int kOffQ = 0;                        // Q_A, then Q_B
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kVStages * kVBytes;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(PairBarriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  // tensor-memory columns of tile t's S (P) and O
  static __device__ __forceinline__ uint32_t col_s(int t) { return t ? 256u : 0u; }
  static __device__ __forceinline__ uint32_t col_o(int t) { return t ? 384u : 128u; }
  static_assert(kOffBar + kBarBytes + 1024 <= kSmem, "bookkeeping must fit the allocation");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static_assert(kKStages <= 3 && kVStages <= 3, "ring barriers hold 3 stages");
  static_assert(!F8 || D == 128, "FP8 PV takes 128-byte e4m3 rows (d = 128)");
  static_assert(kVBytes % 1024 == 0 && kKVBytes % 1024 == 0, "swizzled tiles stay 1024-aligned");
};


// Walks the ascending union of two CSR rows, one block per call.
struct UnionWalk {
  const int32_t* a;
  const int32_t* b;
  int na, nb, ia = 0, ib = 0;
  __device__ __forceinline__ int next(bool& in_a, bool& in_b) {
    const int ca = ia < na ? __ldg(a + ia) : 0x7fffffff;
    const int cb = ib < nb ? __ldg(b + ib) : 0x7fffffff;
    const int c = ca < cb ? ca : cb;
    in_a = ca == c && ia < na;
    in_b = cb == c && ib < nb;
    ia += in_a;
    ib += in_b;
    return c;
  }
};

// F8: the PV product in FP8 (kind::f8f6f4): P rounded to e4m3 (scaled by 2^6
// through the exponent, with the lazy re-basing threshold lowered to 2^2 so P
// stays below 2^8 < 448 and mostly above e4m3's subnormal range) times V in
// e4m3 with one scale per (head, channel); QK^T stays bf16.
template <int D, int BK, bool F8 = false>
__global__ void __launch_bounds__(kPairThreads, 1)
    sparse_attention_pair_kernel(const __grid_constant__ AttnParams p) {
  using C = PairCfg<D, BK, F8>;
  constexpr float kRebase = F8 ? kRebaseLog2F8 : kRebaseLog2;
  constexpr float kPShift = F8 ? kPShiftLog2F8 : 0.0f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  PairBarriers* bar = reinterpret_cast<PairBarriers*>(smem + C::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  // Work order (1-D grid): first the pairs holding text rows (dense rows, by far
  // the longest) of every head, so none of them starts near the end; then the
  // remaining pairs head by head, last pair first, so the CTAs running at the
  // same time share one head's K/V window in L2.
  const int npairs = (p.nqb + 1) >> 1;
  const int first_text_pair = (p.Nv / 128) >> 1;  // pair holding the first text row
  const int n_long = npairs - first_text_pair;
  const int lin = static_cast<int>(blockIdx.x);
  int pair, bh;
  if (lin < n_long * p.BH) {
    bh = lin % p.BH;
    pair = npairs - 1 - lin / p.BH;
  } else {
    const int rest = lin - n_long * p.BH;
    const int per_head = npairs - n_long;
    bh = rest / per_head;
    pair = per_head - 1 - rest % per_head;
  }

  const int label = p.labels ? static_cast<int>(p.labels[bh]) : SVG_HEAD_SPATIAL;
  const int sel = label == SVG_HEAD_TEMPORAL ? 1 : 0;
  if ((label != SVG_HEAD_SPATIAL && label != SVG_HEAD_TEMPORAL) ||
      (sel == 1 && !p.has_permuted && !p.gather)) {
    if (tid == 0) atomicOr(p.status, kDevErrBounds);
    return;
  }
  // Temporal heads of the fused layout path: query rows gathered in
  // position-major order from the frame-major q, outputs scattered back; key
  // and value rows gathered too, or read from position-major copies.
  const bool gather = p.gather != 0 && sel == 1;
  const bool gather_kv = gather && p.gather_kv != 0;
  // CSR rows of the two tiles (tile B may not exist at an odd tail)
  int qb[2], nt[2];
  const int32_t* cols[2];
  for (int t = 0; t < 2; ++t) {
    qb[t] = 2 * pair + t;
    nt[t] = 0;
    cols[t] = p.col_idx[sel];
    if (qb[t] < p.nqb) {
      const int csr_row = (p.csr_per_head ? bh * p.nqb : 0) + qb[t];
      const int32_t r0 = __ldg(p.row_ptr[sel] + csr_row);
      int32_t len = __ldg(p.row_ptr[sel] + csr_row + 1) - r0;
      if (len < 0 || len > p.nkb) {
        if (tid == 0) atomicOr(p.status, kDevErrBounds);
        len = 0;
      }
      nt[t] = len;
      cols[t] = p.col_idx[sel] + r0;
    }
  }

  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar->s_full[t], 1);
      mbar_init(&bar->p_full[t], 128);
      mbar_init(&bar->o_final[t], 1);
    }
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const bool any_work = nt[0] > 0 || nt[1] > 0;

  if (warp >= 8) {
    // producer / MMA warpgroup: hand registers to the softmax warpgroups
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairOtherRegs));
    if (warp == kPairProducerWarp) {
      // ------------------------------------------------------------ producer
      // Lane 0 waits and posts the byte counts. Tiled loads come from lane 0;
      // row gathers (temporal heads of the fused layout path) from lanes
      // 0..rows/4-1, four rows each per 64-column panel.
      const int lane = lane_id();
      if (any_work) {
        const CUtensorMap* mq = &p.tm_q[sel];
        const CUtensorMap* mk = &p.tm_k[sel];
        const CUtensorMap* mv = &p.tm_v[sel];
        const uint64_t keep = l2_policy_evict_last();
        // Rows j0 .. j0+nrows-1 (position-major) of head bh -> dst, a tile of
        // nrows x 128 B panels, panel stride `panel`.
        auto gather_rows = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* b, int j0,
                               int nrows, int panel, uint64_t policy) {
          const int r = 4 * lane;
          if (r >= nrows) return;
          int src[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            src[i] = bh * p.N + frame_major_row(j0 + r + i, p.N, p.Nv, p.T, p.P);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_gather4_hint(dst + pn * panel + r * 128, map, b, pn * 64, src[0], src[1], src[2],
                             src[3], policy);
        };
        uint32_t qbytes = 0;
        for (int t = 0; t < 2; ++t) qbytes += nt[t] > 0 ? C::kQBytes : 0;
        if (lane == 0) mbar_arrive_expect_tx(&bar->q_full, qbytes);
        __syncwarp();
        for (int t = 0; t < 2; ++t) {
          if (nt[t] == 0) continue;
          if (gather) {
            gather_rows(sQ + t * C::kQBytes, mq, &bar->q_full, qb[t] * 128, 128, C::kQPanel, keep);
          } else if (lane == 0) {
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(sQ + t * C::kQBytes + pn * C::kQPanel, mq, &bar->q_full, pn * 64,
                          qb[t] * 128, bh);
          }
        }
        UnionWalk walk{cols[0], cols[1], nt[0], nt[1]};
        int issued = 0;
        for (int u = 0;; ++u) {
          bool ia, ib;
          int c = walk.next(ia, ib);
          if (!ia && !ib) break;
          if (c < 0 || c >= p.nkb) c = 0;  // flagged and masked by the softmax warps
          const int sk = u % C::kKStages;
          const int sv = u % C::kVStages;
          bool ok = true;
          if (lane == 0) {
            ok = mbar_wait(&bar->k_empty[sk], ((u / C::kKStages) & 1) ^ 1, abort_flag, p.status);
            if (ok) mbar_arrive_expect_tx(&bar->k_full[sk], C::kKVBytes);
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
          if (gather_kv) {
            gather_rows(sK + sk * C::kKVBytes, mk, &bar->k_full[sk], c * BK, BK, C::kKVPanel, keep);
          } else if (lane == 0) {
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d_hint(sK + sk * C::kKVBytes + pn * C::kKVPanel, mk, &bar->k_full[sk],
                               pn * 64, c * BK, bh, keep);
          }
          if (lane == 0) {
            ok = mbar_wait(&bar->v_empty[sv], ((u / C::kVStages) & 1) ^ 1, abort_flag, p.status);
            if (ok) mbar_arrive_expect_tx(&bar->v_full[sv], C::kVBytes);
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) {
            issued = -(u + 1);  // K of step u is in flight, V is not
            break;
          }
          if constexpr (F8) {
            if (lane == 0)
              tma_load_3d_hint(sV + sv * C::kVBytes, &p.tm_v8, &bar->v_full[sv], 0, c * BK, bh, keep);
          } else if (gather_kv) {
            gather_rows(sV + sv * C::kVBytes, mv, &bar->v_full[sv], c * BK, BK, C::kKVPanel, keep);
          } else if (lane == 0) {
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d_hint(sV + sv * C::kVBytes + pn * C::kKVPanel, mv, &bar->v_full[sv],
                               pn * 64, c * BK, bh, keep);
          }
          issued = u + 1;
        }
        if (lane == 0 && *abort_flag) {
          // Let every copy this warp started land before the CTA retires.
          const int done = issued < 0 ? -issued : issued;
          for (int u = (done > C::kKStages ? done - C::kKStages : 0); u < done; ++u) {
            long long t0 = clock64();
            while (!mbar_try_wait(&bar->k_full[u % C::kKStages], (u / C::kKStages) & 1) &&
                   clock64() - t0 < kWaitLimitCycles) {
            }
          }
          const int v_done = issued >= 0 ? done : done - 1;
          for (int u = (v_done > C::kVStages ? v_done - C::kVStages : 0); u < v_done; ++u) {
            long long t0 = clock64();
            while (!mbar_try_wait(&bar->v_full[u % C::kVStages], (u / C::kVStages) & 1) &&
                   clock64() - t0 < kWaitLimitCycles) {
            }
          }
        }
      }
    } else if (warp == kPairMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      if (lane_id() == 0 && any_work) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BK, false, false);
        constexpr uint32_t idesc_pv =
            F8 ? idesc_e4m3_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
        const uint32_t q_addr = smem_u32(sQ);
        const uint32_t k_addr = smem_u32(sK);
        const uint32_t v_addr = smem_u32(sV);
        bool ok = mbar_wait(&bar->q_full, 0, abort_flag, p.status);
        tc_fence_after();
        UnionWalk walk{cols[0], cols[1], nt[0], nt[1]};
        bool prev_in[2] = {false, false};
        int pv_done[2] = {0, 0};
        for (int u = 0; ok; ++u) {
          bool in[2];
          walk.next(in[0], in[1]);
          const bool step = in[0] || in[1];  // false: drain step after the last block
          if (!step && !prev_in[0] && !prev_in[1]) break;
          const int st = u % C::kKStages;
          const int pst = (u + C::kVStages - 1) % C::kVStages;
          bool k_ready = false, v_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (prev_in[t]) {  // PV_t of the previous step
              if (!v_ready) {
                ok = mbar_wait(&bar->v_full[pst], ((u - 1) / C::kVStages) & 1, abort_flag, p.status);
                v_ready = true;
              }
              if (ok) ok = mbar_wait(&bar->p_full[t], pv_done[t] & 1, abort_flag, p.status);
              if (!ok) break;
              tc_fence_after();
              if constexpr (F8) {
                // K = 32 keys per MMA: 8 tensor-memory columns of four e4m3 P values,
                // 32 rows of 128 e4m3 V bytes (one 128-byte swizzle atom across d)
  #pragma unroll
                for (int kk = 0; kk < BK / 32; ++kk) {
                  const uint64_t b = sdesc_sw128(v_addr + pst * C::kVBytes + kk * 32 * 128,
                                                 C::kVBytes, 1024);
                  mma_f8_ts(tmem + C::col_o(t), tmem + C::col_s(t) + kk * 8, b, idesc_pv,
                            (pv_done[t] > 0 || kk > 0) ? 1u : 0u);
                }
              } else {
  #pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                  const uint64_t b = sdesc_sw128(v_addr + pst * C::kVBytes + kk * 16 * 128,
                                                 C::kKVPanel, 1024);
                  mma_bf16_ts(tmem + C::col_o(t), tmem + C::col_s(t) + kk * 8, b, idesc_pv,
                              (pv_done[t] > 0 || kk > 0) ? 1u : 0u);
                }
              }
              ++pv_done[t];
              if (pv_done[t] == nt[t]) tc_commit(&bar->o_final[t]);
            }
            if (step && in[t]) {  // QK_t of this step
              if (!k_ready) {
                ok = mbar_wait(&bar->k_full[st], (u / C::kKStages) & 1, abort_flag, p.status);
                k_ready = true;
                if (!ok) break;
              }
              tc_fence_after();
  #pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t a = sdesc_sw128(q_addr + t * C::kQBytes + (kk >> 2) * C::kQPanel + off,
                                               16, 1024);
                const uint64_t b = sdesc_sw128(
                    k_addr + st * C::kKVBytes + (kk >> 2) * C::kKVPanel + off, 16, 1024);
                mma_bf16_ss(tmem + C::col_s(t), a, b, idesc_qk, kk > 0 ? 1u : 0u);
              }
              tc_commit(&bar->s_full[t]);
            }
          }
          if (!ok) break;
          if (u >= 1) tc_commit(&bar->v_empty[pst]);
          if (step) tc_commit(&bar->k_empty[st]);
          prev_in[0] = in[0];
          prev_in[1] = in[1];
          if (!step) break;
        }
        if (*abort_flag) {
          tc_commit(&bar->drain);
          long long t0 = clock64();
          while (!mbar_try_wait(&bar->drain, 0) && clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairSoftmaxRegs));
    // ------------------------------------------------------------ softmax (tile t)
    const int t = warp >> 2;
    const int r = tid & 127;  // row within the tile = TMEM lane
    const int row = qb[t] * 128 + r;
    const bool row_valid = qb[t] < p.nqb && row < p.N;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = lane_base + C::col_s(t);
    const uint32_t o_col = lane_base + C::col_o(t);
    const int n = nt[t];
    const int32_t* my_cols = cols[t];
    float m = -INFINITY;  // running base, log2 units
    float l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int c = __ldg(my_cols + j);
      const bool bad = c < 0 || c >= p.nkb;
      if (bad && r == 0) atomicOr(p.status, kDevErrBounds);
      int kvalid = bad ? 0 : p.N - c * BK;
      if (kvalid > BK) kvalid = BK;
      if (!mbar_wait(&bar->s_full[t], j & 1, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[BK];
#pragma unroll
      for (int ch = 0; ch < BK / 32; ++ch)
        tmem_ld_32x32b_x32(s_col + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      tmem_ld_wait();
      reg_fence(sr);
      if (kvalid < BK) {  // the ragged last key block (or a flagged index)
#pragma unroll
        for (int i = 0; i < BK; ++i)
          if (i >= kvalid) sr[i] = __float_as_uint(-INFINITY);
      }
      // row maximum: eight independent 3-input max chains, then a small tree
      float xm[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) xm[c] = fmax3(u2f(sr[2 * c]), u2f(sr[2 * c + 1]), -INFINITY);
#pragma unroll
      for (int i = 16; i < BK; i += 16) {
#pragma unroll
        for (int c = 0; c < 8; ++c) xm[c] = fmax3(xm[c], u2f(sr[i + 2 * c]), u2f(sr[i + 2 * c + 1]));
      }
      const float m_tile =
          fmaxf(fmax3(xm[0], xm[1], xm[2]), fmax3(xm[3], fmax3(xm[4], xm[5], xm[6]), xm[7])) *
          p.scale_log2;
      const bool rebase = m_tile > m + kRebase;
      const float m_new = rebase ? m_tile : m;
      const float alpha = rebase ? fast_exp2(m - m_new) : 1.0f;  // exp2(-inf) = 0
      // FP8: the probabilities (and so the row sum) carry a factor 2^kPShift
      const float m_use = (m_new == -INFINITY ? 0.0f : m_new) - kPShift;
      float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
      for (int ch = 0; ch < BK / 32; ++ch) {
        if constexpr (F8) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c0 = ch * 32 + 4 * i;
            float y0, y1, y2, y3;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -m_use, -m_use);
            ffma2(y2, y3, u2f(sr[c0 + 2]), u2f(sr[c0 + 3]), p.scale_log2, p.scale_log2, -m_use,
                  -m_use);
            const float e0 = fast_exp2(y0), e1 = fast_exp2(y1);
            const float e2 = fast_exp2(y2), e3 = fast_exp2(y3);
            fadd2(s0, s1, s0, s1, e0, e1);
            fadd2(s0, s1, s0, s1, e2, e3);
            pk[i] = pack_e4m3x4(e0, e1, e2, e3);
          }
          tmem_st_32x32b_x8(s_col + ch * 8, pk);
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = ch * 32 + 2 * i;
            float y0, y1;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -m_use, -m_use);
            const float e0 = fast_exp2(y0);
            const float e1 = fast_exp2(y1);
            fadd2(s0, s1, s0, s1, e0, e1);
            pk[i] = pack_bf16x2(e0, e1);
          }
          tmem_st_32x32b_x16(s_col + ch * 16, pk);
        }
      }
      l = l * alpha + (s0 + s1);
      m = m_new;
      tmem_st_wait();
      // PV_t(j-1) retired with QK_t(j), so O_t may be re-based right away.
      if (j > 0 && __any_sync(0xffffffffu, rebase)) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(o_col + ch * 32, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * alpha);
          tmem_st_32x32b_x32(o_col + ch * 32, o);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[t]);
    }

    // ---- epilogue: O / l -> bf16, lse
    if (ok && n > 0) ok = mbar_wait(&bar->o_final[t], 0, abort_flag, p.status);
    tc_fence_after();
    const bool have_o = __all_sync(0xffffffffu, ok) && n > 0;
    // the fused layout path writes temporal rows straight to their frame-major place
    const int out_row = gather && row_valid ? frame_major_row(row, p.N, p.Nv, p.T, p.P) : row;
    svg_bf16* out = p.out[sel] + (static_cast<size_t>(bh) * p.N + out_row) * D;
    const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld_32x32b_x32(o_col + ch * 32, o);
        tmem_ld_wait();
        reg_fence(o);
      }
      if constexpr (F8) {  // undo V's per-channel quantisation scale
        const float* vs = p.v_scale + static_cast<size_t>(bh) * D + ch * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * __ldg(vs + i));
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = have_o ? pack_bf16x2(u2f(o[2 * i]) * inv_l, u2f(o[2 * i + 1]) * inv_l) : 0u;
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + ch * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
    }
    if (p.lse != nullptr && row_valid) {
      p.lse[static_cast<size_t>(bh) * p.N + out_row] =
          (have_o && l > 0.0f) ? (m + __log2f(l) - kPShift) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, int BK>
cudaError_t launch_impl(const Dims& d, const AttnParams& p, cudaStream_t stream);

template <int D, int BK, bool F8 = false>
cudaError_t launch_pair(const Dims& d, const AttnParams& p, cudaStream_t stream) {
  using C = PairCfg<D, BK, F8>;
  auto kern = sparse_attention_pair_kernel<D, BK, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  // The register hand-over inside the kernel is only balanced when the kernel
  // launches at exactly kPairLaunchRegs per thread; otherwise (or if a CTA
  // cannot be resident) use the single-tile kernel.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  int resident = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, kPairThreads, C::kSmem);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kPairLaunchRegs || resident < 1) {
    // the single-tile kernel has no row gathers and no FP8 product
    if (p.gather || F8) return cudaErrorNotSupported;
    return launch_impl<D, BK>(d, p, stream);
  }
  dim3 grid(static_cast<unsigned>(((d.nqb + 1) / 2) * d.BH));
  kern<<<grid, kPairThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_impl(const Dims& d, const AttnParams& p, cudaStream_t stream) {
  using C = Cfg<D, BK>;
  auto kern = sparse_attention_kernel<D, BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(d.nqb, d.BH);
  kern<<<grid, kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attention(const Dims& d, const AttnArgs& a, int* status,
                                    cudaStream_t stream) {
  AttnParams p;
  memset(&p, 0, sizeof(p));
  const bool f8 = a.v8 != nullptr;
  const bool perm = a.qp != nullptr && !a.fused;
  if (a.fused && d.bq != 128) return cudaErrorNotSupported;
  if (f8 && (d.bq != 128 || d.d != 128 || a.fused)) return cudaErrorNotSupported;
  if (!make_tmap_bf16(&p.tm_q[0], a.q, d.d, d.N, d.BH, d.bq) ||
      !make_tmap_bf16(&p.tm_k[0], a.k, d.d, d.N, d.BH, d.bk))
    return cudaErrorInvalidValue;
  if (f8) {
    if (!make_tmap_u8_rows128(&p.tm_v8, a.v8, d.N, d.BH, d.bk)) return cudaErrorInvalidValue;
    p.v_scale = a.v_scale;
    p.tm_v[0] = p.tm_k[0];  // unused by the FP8 product
  } else if (!make_tmap_bf16(&p.tm_v[0], a.v, d.d, d.N, d.BH, d.bk)) {
    return cudaErrorInvalidValue;
  }
  if (a.fused) {
    const int64_t rows = static_cast<int64_t>(d.BH) * d.N;
    if (!make_tmap_rows_bf16(&p.tm_q[1], a.q, d.d, rows)) return cudaErrorInvalidValue;
    if (a.kp != nullptr) {  // position-major copies of K and V
      if (!make_tmap_bf16(&p.tm_k[1], a.kp, d.d, d.N, d.BH, d.bk) ||
          !make_tmap_bf16(&p.tm_v[1], a.vp, d.d, d.N, d.BH, d.bk))
        return cudaErrorInvalidValue;
    } else if (!make_tmap_rows_bf16(&p.tm_k[1], a.k, d.d, rows) ||
               !make_tmap_rows_bf16(&p.tm_v[1], a.v, d.d, rows)) {
      return cudaErrorInvalidValue;
    }
  } else if (perm) {
    if (!make_tmap_bf16(&p.tm_q[1], a.qp, d.d, d.N, d.BH, d.bq) ||
        !make_tmap_bf16(&p.tm_k[1], a.kp, d.d, d.N, d.BH, d.bk))
      return cudaErrorInvalidValue;
    if (f8) {
      p.tm_v[1] = p.tm_k[1];  // unused by the FP8 product
    } else if (!make_tmap_bf16(&p.tm_v[1], a.vp, d.d, d.N, d.BH, d.bk)) {
      return cudaErrorInvalidValue;
    }
  } else {
    p.tm_q[1] = p.tm_q[0];
    p.tm_k[1] = p.tm_k[0];
    p.tm_v[1] = p.tm_v[0];
  }
  p.labels = a.labels;
  p.row_ptr[0] = a.row_ptr_s;
  p.col_idx[0] = a.col_idx_s;
  p.row_ptr[1] = a.row_ptr_t ? a.row_ptr_t : a.row_ptr_s;
  p.col_idx[1] = a.col_idx_t ? a.col_idx_t : a.col_idx_s;
  p.out[0] = a.o;
  p.out[1] = a.op && !a.fused ? a.op : a.o;
  p.lse = a.lse;
  p.status = status;
  p.N = d.N;
  p.Nv = d.Nv;
  p.BH = d.BH;
  p.nqb = d.nqb;
  p.nkb = d.nkb;
  p.bq = d.bq;
  p.bk = d.bk;
  p.has_permuted = perm && a.op != nullptr && a.row_ptr_t != nullptr && a.col_idx_t != nullptr;
  p.csr_per_head = a.csr_per_head ? 1 : 0;
  p.gather = a.fused ? 1 : 0;
  p.gather_kv = a.fused && a.kp == nullptr ? 1 : 0;
  p.T = d.T;
  p.P = d.P;
  p.scale_log2 = d.scale * 1.4426950408889634f;
  if (f8) {
    if (d.bk == 128) return launch_pair<128, 128, true>(d, p, stream);
    return launch_pair<128, 64, true>(d, p, stream);
  }
  if (d.bq == 128) {
    if (d.d == 128 && d.bk == 128) return launch_pair<128, 128>(d, p, stream);
    if (d.d == 128 && d.bk == 64) return launch_pair<128, 64>(d, p, stream);
    if (d.d == 64 && d.bk == 128) return launch_pair<64, 128>(d, p, stream);
    return launch_pair<64, 64>(d, p, stream);
  }
  if (d.d == 128 && d.bk == 128) return launch_impl<128, 128>(d, p, stream);
  if (d.d == 128 && d.bk == 64) return launch_impl<128, 64>(d, p, stream);
  if (d.d == 64 && d.bk == 128) return launch_impl<64, 128>(d, p, stream);
  return launch_impl<64, 64>(d, p, stream);
}

}  // namespace svg
