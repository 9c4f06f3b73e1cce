// Attention over the selected latent rows on tcgen05 tensor cores, for
// launches with many query rows (prefill).
//
//   O[q, g, :] = sum_{s in S_q} softmax_s( scale * q[q, g, :] . kv[s, :] ) * kv[s, :512]
//
// (llama.cpp b12180 news: aiaulis.com paragraph 2 — attention only over the
// selected tokens; devotd.net section 2 — one key-only latent cache whose
// leading 512 entries serve as V.)
//
// One CTA owns one query row and a block of 64 heads, and walks the row's
// selected set in tiles of 48 gathered cache rows:
//   S    = Q[64 heads, 576] . K_tile[48, 576]^T      M = 64,  N = 48, K = 576
//   O^T += V_tile^T[512, 48] . P^T[48, 64 heads]     M = 128 (x4), N = 64, K = 48
// Q's first 384 dims sit in TMEM for the whole row, so the S products read
// that part of their A operand from tensor memory and only the last 192 dims
// from shared memory; the shared memory this frees holds a third gather
// stage.  S lands in TMEM with one head per lane, so each softmax thread
// owns one head row: max, exp2 and row sum stay in registers.  P is written to shared
// memory as bf16 hi + lo parts (two MMAs), keeping its rounding error near
// 2^-16, on rows with fewer than kHiOnlyRows selected; longer rows take the
// hi part alone.  The gathered tile is stored once, in the 128-byte swizzled layout,
// and read by both MMAs: K-major as the B operand of S, MN-major as the A
// operand of O^T.  The running maximum is raised lazily (only when a tile's
// maximum exceeds it by more than 2^8), and O^T in TMEM is then rescaled.
//
// Warp roles (352 threads): warps 0-3 softmax and output (TMEM quadrants
// 0-3), warp 4 TMEM allocation, the Q load (TMA) and single-thread MMA issue,
// warps 5-6, 7-8 and 9-10 gather tiles t = 0, 1, 2 (mod 3) with 16-byte
// cp.async into three stages.  A stage is busy from its gather until its
// tile's P.V completes (gather, S, softmax, P.V in a chain), so three stages
// keep more of that chain in flight than two; the tensor core's cost per
// product (about the same for N = 32 as for N = 48) makes the larger tile
// the cheaper one per key.
//
// The same kernel, instantiated with kMasked, is the mask-over-the-whole-
// cache route the pages describe for llama.cpp (aiaulis.com paragraph 4;
// devotd.net section 2: the selection becomes a mask so that the existing
// sparse flash attention is reused): a CTA owns a chunk of the row's causal
// positions instead of a slice of its index set, streams every cached row of
// the chunk with TMA tile loads, and masks the logits of the rows that the
// index set does not list (a bitmap of the chunk built from it).  It reads
// the whole latent cache; it is kept as the measured comparison to the
// gather.
#include <algorithm>

#include "attn_tc_common.cuh"

namespace dsa {
namespace {

using namespace attn_tc;

constexpr int kT = 48;                    // gathered rows per tile
constexpr int kStages = 3;                // gather stages
constexpr int kSBufs = 1;                 // S buffers in TMEM
constexpr int kPStages = 2;               // P buffers
constexpr int kHB = 64;                   // heads per CTA
constexpr int kBoxes = kLatent / 64;      // 64-dim column boxes of a latent row
constexpr int kQBox = kHB * 128;          // bytes of one Q box
constexpr int kQTmemBoxes = 6;            // Q dims 0..383: TMEM (A operand of S)
constexpr int kQSmemBoxes = kBoxes - kQTmemBoxes;  // Q dims 384..575: shared memory
constexpr int kKVBox = kT * 128;          // bytes of one gathered-tile box
constexpr int kKVStage = kBoxes * kKVBox;
constexpr int kPBuf = kHB * 128;          // one P operand (64 heads x 64 keys, 48 used)
constexpr int kSoftThreads = 128;
constexpr int kGroupThreads = 64;         // one gather group
constexpr int kThreadsTc = kSoftThreads + 32 + kStages * kGroupThreads;
constexpr float kRescaleLog2 = 8.0f;      // raise the running max only past 2^8
// Rows with at least this many selected slots take P as bf16 alone (no lo
// part): the weights of so many keys are spread thin enough that their
// rounding stays inside the output tolerance of 2e-3 (largest errors seen on
// N(0,1) latents: 9.2e-4 over 40 rows x 80 heads at 1024 keys, 5.5e-4 over
// 48 rows x 64 heads at 2048), and the row sum is taken over the rounded
// values, so the weights still sum to one.
constexpr int kHiOnlyRows = 1024;

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQSmemBoxes * kQBox;
constexpr int kOffStage = kOffQ;  // output staging [64][512] fp32 over Q and the gather stages
constexpr int kOffP = kOffKV + kStages * kKVStage;     // [P stage][hi, lo]
constexpr int kOffBar = kOffP + 2 * kPStages * kPBuf;
constexpr int kNumBars = 4 + 2 * kStages + 2 * kSBufs + 2 * kPStages;
constexpr int kOffTmem = kOffBar + 8 * kNumBars;
constexpr int kOffIdx = kOffTmem + 16;                  // [kStages][kT] int
constexpr int kOffAlpha = kOffIdx + kStages * kT * 4;   // [64] float
constexpr int kOffM = kOffAlpha + kHB * 4;              // [64] float
constexpr int kOffL = kOffM + kHB * 4;                  // [64] float
constexpr int kOffMask = kOffL + kHB * 4;               // masked route: chunk bitmap
constexpr int kMaskWords = 1024;                        // positions per chunk <= 32768
constexpr int kSmemUsed = kOffMask + kMaskWords * 4;
constexpr int kSmemTc = kSmemUsed + 1024;               // alignment slack
static_assert(kOffStage + kHB * kValue * 4 <= kOffP, "output staging overlaps the P buffers");
static_assert(kSmemTc <= 227 * 1024, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // the S buffer, columns 0..47 (M = 64 layout)
constexpr uint32_t kColQ = 64;    // Q dims 0..383, two bf16 per column (M = 64 layout)
constexpr uint32_t kColO = 256;   // O^T blocks at 256, 320, 384, 448
static_assert(kColS + kT * kSBufs <= kColQ && kColQ + 32 * kQTmemBoxes <= kColO &&
                  kColO + 4 * 64 <= kTmemCols,
              "TMEM columns");

// kind::f16 instruction descriptors (bf16 in, fp32 accumulate).
constexpr uint32_t kIdescS = idesc_bf16_f32(64, kT);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHB) | (1u << 15);  // A MN-major
constexpr int kSplitCols = kT / 2;  // logits per half warp (16 + 8 columns)
static_assert(kSplitCols == 24, "the logit loads cover 16 + 8 columns per half warp");

template <bool kMasked>
__global__ void __launch_bounds__(kThreadsTc, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap kvmap, const TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const bp = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sKV = base + kOffKV, sP = base + kOffP;
  const uint32_t bars = base + kOffBar;
  const uint32_t b_qfull = bars;
  auto b_kvfull = [&](int s) { return bars + 8u * (1 + s); };
  auto b_kvempty = [&](int s) { return bars + 8u * (1 + kStages + s); };
  auto b_sfull = [&](int s) { return bars + 8u * (1 + 2 * kStages + s); };
  auto b_sempty = [&](int s) { return bars + 8u * (1 + 2 * kStages + kSBufs + s); };
  auto b_pfull = [&](int s) { return bars + 8u * (1 + 2 * kStages + 2 * kSBufs + s); };
  auto b_pempty = [&](int s) { return bars + 8u * (1 + 2 * kStages + 2 * kSBufs + kPStages + s); };
  const uint32_t b_odone = bars + 8u * (1 + 2 * kStages + 2 * kSBufs + 2 * kPStages);
  const uint32_t b_drain = b_odone + 8u;
  const uint32_t b_qtmem = b_odone + 16u;  // Q's TMEM part stored
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bp + kOffTmem);
  int* const tidx = reinterpret_cast<int*>(bp + kOffIdx);
  float* const alpha_s = reinterpret_cast<float*>(bp + kOffAlpha);
  float* const rl_s = reinterpret_cast<float*>(bp + kOffL);  // 1 / row sum per head
  uint32_t* const mask = reinterpret_cast<uint32_t*>(bp + kOffMask);

  const int warp = warp_id_uniform();
  const int lane = lane_id();
  const int r = blockIdx.x;
  const int h0 = blockIdx.y * kHB;
  const int sp = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b_kvfull(s), kMasked ? 1 : kGroupThreads);
      mbar_init(b_kvempty(s), 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(b_sfull(s), 1);
      mbar_init(b_sempty(s), kSoftThreads);
    }
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(b_pfull(s), kSoftThreads);
      mbar_init(b_pempty(s), 1);
    }
    mbar_init(b_odone, 1);
    mbar_init(b_drain, 1);
    mbar_init(b_qtmem, kSoftThreads);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();
  pdl_launch_dependents();
  const RowSeq rs = row_seq_warp(P.q_offsets, P.cache, P.ctx_lens, P.B, r);
  const long long kv0 = rs.rows.kv0;  // the masked route's contiguous rows
  const int32_t* const idx_row = P.idx + static_cast<size_t>(r) * P.top_k;
  // With idx_prefix, slots past min(top_k, p+1) hold -1: skip their tiles.
  const int n_slots = P.idx_prefix ? min(P.top_k, rs.len) : P.top_k;
  // This CTA's slice of the slots (of the causal positions, masked route).
  const int slot_lo = sp * P.split_len;
  const int slot_hi = min(kMasked ? rs.len : n_slots, slot_lo + P.split_len);
  const int n_tiles = slot_hi > slot_lo ? (slot_hi - slot_lo + kT - 1) / kT : 0;
  // The lo part of P only for rows with fewer than kHiOnlyRows selected.
  const bool use_lo = min(P.top_k, rs.len) < kHiOnlyRows;
  if (kMasked) {
    // Bitmap of the chunk's positions that the index set lists.
    const int nwords = (P.split_len + 31) >> 5;
    for (int i = threadIdx.x; i < nwords; i += kThreadsTc) mask[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < P.top_k; i += kThreadsTc) {
      const int pos = __ldg(idx_row + i);
      if (pos < -1 || pos >= rs.len) {  // outside 0..p: skipped and recorded
        atomicOr(P.err, kErrIndex);
      } else if (pos >= slot_lo && pos < slot_hi) {
        atomicOr(&mask[(pos - slot_lo) >> 5], 1u << ((pos - slot_lo) & 31));
      }
    }
    __syncthreads();
  }

  if (kMasked && warp >= 5) {
    // ----------------------------------------- whole-cache tiles (masked) --
    // Each group stages its tiles' positions (-1 where the mask drops the row)
    // and one thread loads all rows of the tile with TMA.
    const int grp = (warp - 5) >> 1;
    const int gt = threadIdx.x - (5 + 2 * grp) * 32;
    int* const gidx = tidx + grp * kT;
    const uint64_t pol = l2_policy_evict_first();
    bool ok = true;
    int last_t = -1;  // the last tile this group loaded
    for (int t = grp; t < n_tiles && ok; t += kStages) {
      const uint32_t ph = static_cast<uint32_t>((t / kStages) & 1);
      ok = mbar_wait(b_kvempty(grp), ph ^ 1u, P.err);
      if (!ok) break;
      if (gt < kT) {
        const int rel = t * kT + gt;
        const int pos = slot_lo + rel;
        const bool on = pos < slot_hi && ((mask[rel >> 5] >> (rel & 31)) & 1u);
        gidx[gt] = on ? pos : -1;
      }
      named_bar_sync(2 + grp, kGroupThreads);
      if (gt == 0) {
        const uint32_t stage = sKV + grp * kKVStage;
        mbar_arrive_expect_tx(b_kvfull(grp), kKVStage);
        const int row = static_cast<int>(kv0 + slot_lo + t * kT);
        for (int bx = 0; bx < kBoxes; ++bx) {
          tma_load_2d(stage + bx * kKVBox, &kvmap, b_kvfull(grp), 64 * bx, row, pol);
        }
        last_t = t;
      }
    }
    // The loads this group issued land before the CTA may exit.
    if (gt == 0 && last_t >= 0) {
      mbar_drain(b_kvfull(grp), static_cast<uint32_t>((last_t / kStages) & 1), P.err);
    }
  } else if (warp >= 5) {
    // ------------------------------------------------------------ gather --
    // The group copies the tile's rows in 16-byte pieces with the swizzle
    // applied, after it has staged the tile's positions.
    const int grp = (warp - 5) >> 1;            // tiles t = grp (mod kStages)
    const int gt = threadIdx.x - (5 + 2 * grp) * 32;
    int* const gidx = tidx + grp * kT;
    // Cache rows of tile t's slots (thread gt < kT holds one), loaded and
    // prefetched into L2 a tile ahead of their copy.
    auto load_row = [&](int t) -> int {
      if (gt >= kT || t >= n_tiles) return -1;
      const int slot = slot_lo + t * kT + gt;
      if (slot >= slot_hi) return -1;
      const int pos = __ldg(idx_row + slot);
      // Only positions 0..p of the row are read; any other entry but -1 is
      // recorded as an error and skipped.
      if (pos < -1 || pos >= rs.len) {
        atomicOr(P.err, kErrIndex);
        return -1;
      }
      // The slot's cache row (-1: nothing to read).
      return pos >= 0 ? static_cast<int>(seq_row(rs.rows, pos)) : -1;
    };
    auto prefetch_row = [&](int row) {
      if (row >= 0) {
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                         P.kv + static_cast<size_t>(row) * kLatent),
                     "r"(kLatent * 2)
                     : "memory");
      }
    };
    // The first tile's rows are copied at once (no prefetch); later tiles'
    // rows are prefetched one of the group's tiles ahead.
    int row_cur = load_row(grp);
    int row_nxt = load_row(grp + kStages);
    bool ok = true;
    for (int t = grp; t < n_tiles && ok; t += kStages) {
      // Later tiles prefetch while they wait for their stage; the first
      // does so after its copies have landed (it waits on nothing before).
      if (t != grp) prefetch_row(row_nxt);
      const uint32_t ph = static_cast<uint32_t>((t / kStages) & 1);
      ok = mbar_wait(b_kvempty(grp), ph ^ 1u, P.err);
      if (!ok) break;
      if (gt < kT) gidx[gt] = row_cur;
      named_bar_sync(2 + grp, kGroupThreads);
      row_cur = row_nxt;
      const uint32_t stage = sKV + grp * kKVStage;
      // Thread (sub, piece) copies 16-byte piece `piece` of every box of
      // rows sub, sub + 8, ...: a warp instruction reads four whole 128-byte
      // lines, its four swizzled rows cover every shared-memory bank four
      // times, and the swizzle (row & 7 == sub) is fixed per thread.
      const uint32_t piece = static_cast<uint32_t>(gt & 7);
      const int sub = gt >> 3;
      const uint32_t sw = (piece ^ static_cast<uint32_t>(sub)) << 4;
      for (int i = sub; i < kT; i += kGroupThreads >> 3) {
        const int row = gidx[i];
        const uint32_t dst = stage + i * 128 + sw;
        if (row >= 0) {
          const __nv_bfloat16* src = P.kv + static_cast<size_t>(row) * kLatent + piece * 8;
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx) cp_async16_tc(dst + bx * kKVBox, src + bx * 64);
        } else {
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx) {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + bx * kKVBox),
                         "r"(0u)
                         : "memory");
          }
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      // The group's slot two tiles ahead is looked up while this tile's
      // copies are in flight (its bounds check branches on the loaded entry).
      row_nxt = load_row(t + 2 * kStages);
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      fence_proxy_async_smem();
      mbar_arrive(b_kvfull(grp));
      if (t == grp) prefetch_row(row_cur);  // the group's next tile (row_cur moved on)
    }
    // The CTA of row r + P.wave starts about when this one ends (one CTA per
    // SM, rows dealt in order): once this CTA's rows are all requested, its
    // index row and query block go to L2, so that its first loads do not
    // wait on DRAM.  Bulk prefetches need 16-byte aligned addresses and
    // sizes.
    if (gt == 0 && grp == 0 && ok && P.wave > 0 && gridDim.y == 1 && gridDim.z == 1 &&
        r + P.wave < P.Nq) {
      const int rn = r + P.wave;
      const int32_t* const ip = P.idx + static_cast<size_t>(rn) * P.top_k;
      if ((P.top_k & 3) == 0 && (reinterpret_cast<uintptr_t>(ip) & 15u) == 0) {
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ip),
                     "r"(static_cast<uint32_t>(P.top_k) * 4u)
                     : "memory");
      }
      const __nv_bfloat16* const qp = P.q + static_cast<size_t>(rn) * P.H * kLatent;
      if ((reinterpret_cast<uintptr_t>(qp) & 15u) == 0) {
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(qp),
                     "r"(static_cast<uint32_t>(P.H) * kLatent * 2u)
                     : "memory");
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------ Q load + MMA issue --
    // The whole warp runs the loop (waits and descriptor arithmetic stay
    // warp-uniform); one elected lane issues each MMA and commit.
    if (lane == 0) {
      tma_prefetch_map(&qmap);
      // Only Q's shared-memory part; the softmax warps store the rest in TMEM.
      mbar_arrive_expect_tx(b_qfull, kQSmemBoxes * kQBox);
      const uint64_t pol = l2_policy_evict_first();
      for (int j = kQTmemBoxes; j < kBoxes; ++j) {
        tma_load_2d(sQ + (j - kQTmemBoxes) * kQBox, &qmap, b_qfull, 64 * j, r * P.H + h0, pol);
      }
    }
    __syncwarp();
    // Descriptors of the first K slice of each operand; later slices add
    // their byte offset / 16 to the address field.
    const uint64_t dq = sdesc_sw128(sQ);
    const uint64_t dkv0 = sdesc_sw128(sKV);
    const uint64_t dv0 = sdesc_sw128_mn(sKV, kKVBox);
    const uint64_t dp0 = sdesc_sw128(sP);
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, P.err));
    };
    bool ok = wait_all(b_qfull, 0) && wait_all(b_qtmem, 0);
    tc_fence_after();
    auto issue_pv = [&](int u) {
      const int st = u % kStages;
      const int pb = u % kPStages;
      const uint64_t dv = dv0 + static_cast<uint64_t>((st * kKVStage) >> 4);
      const uint64_t dhi = dp0 + static_cast<uint64_t>((2 * pb * kPBuf) >> 4);
      const uint64_t dlo = dhi + static_cast<uint64_t>(kPBuf >> 4);
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint64_t a = dv + static_cast<uint64_t>(((2 * blk) * kKVBox + kk * 2048) >> 4);
          const uint32_t d = tmem + kColO + 64u * blk;
          const uint64_t ko = static_cast<uint64_t>((kk * 32) >> 4);
          tc_mma_bf16_warp(d, a, dhi + ko, kIdescPV, (u > 0 || kk > 0) ? 1u : 0u);
          if (use_lo) tc_mma_bf16_warp(d, a, dlo + ko, kIdescPV, 1u);
        }
      }
      tc_commit_warp(b_kvempty(st));
      tc_commit_warp(b_pempty(pb));
      tc_commit_warp(b_odone);
    };
    auto p_ready = [&](int u) {
      return mbar_test_wait(b_pfull(u % kPStages), static_cast<uint32_t>((u / kPStages) & 1));
    };
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int st = t % kStages;
      const uint32_t ph = static_cast<uint32_t>((t / kStages) & 1);
      const int sb = t % kSBufs;
      const uint32_t sph = static_cast<uint32_t>((t / kSBufs) & 1);
      // S(t) goes first: the softmax waits on it.  While tile t's rows are
      // still arriving, the previous tile's P.V is issued as soon as its P is
      // ready, which frees its gather stage early.  The polls do not block
      // (a suspending wait on one barrier would hold up the other).
      bool pv_pending = t > 0;
      const long long w0 = clock64();
      for (unsigned it = 1;; ++it) {
        if (__all_sync(0xffffffffu, mbar_test_wait(b_kvfull(st), ph) &&
                                        mbar_test_wait(b_sempty(sb), sph ^ 1u))) {
          break;
        }
        if (pv_pending && __all_sync(0xffffffffu, p_ready(t - 1))) {
          tc_fence_after();
          issue_pv(t - 1);
          pv_pending = false;
        }
        if ((it & 63u) == 0u) {
          const bool late = clock64() - w0 > kWaitCycles;
          if (__any_sync(0xffffffffu, late || *reinterpret_cast<volatile unsigned*>(P.err) != 0u)) {
            if (lane == 0 && late) atomicOr(P.err, kErrTimeout);
            ok = false;
            break;
          }
        }
      }
      if (!ok) break;
      tc_fence_after();
      const uint64_t dk = dkv0 + static_cast<uint64_t>((st * kKVStage) >> 4);
      const uint32_t d = tmem + kColS + static_cast<uint32_t>(kT) * sb;
#pragma unroll
      for (int ks = 0; ks < kLatent / 16; ++ks) {
        const int box = ks >> 2;
        const uint32_t off = (ks & 3) * 32;
        const uint64_t b = dk + static_cast<uint64_t>((box * kKVBox + off) >> 4);
        if (box < kQTmemBoxes) {  // 16 dims = 8 TMEM columns of Q per K step
          tc_mma_bf16_ts_warp(d, tmem + kColQ + 8u * ks, b, kIdescS, ks > 0 ? 1u : 0u);
        } else {
          tc_mma_bf16_warp(d, dq + static_cast<uint64_t>(((box - kQTmemBoxes) * kQBox + off) >> 4),
                           b, kIdescS, 1u);
        }
      }
      tc_commit_warp(b_sfull(sb));
      if (pv_pending) {
        ok = wait_all(b_pfull((t - 1) % kPStages), static_cast<uint32_t>(((t - 1) / kPStages) & 1));
        if (!ok) break;
        tc_fence_after();
        issue_pv(t - 1);
      }
    }
    if (ok && n_tiles > 0 &&
        wait_all(b_pfull((n_tiles - 1) % kPStages),
                 static_cast<uint32_t>(((n_tiles - 1) / kPStages) & 1))) {
      tc_fence_after();
      issue_pv(n_tiles - 1);
    }
    // Nothing this warp issued (the Q load, the MMAs) may still be running
    // when the CTA exits; immediate unless a wait above was abandoned.
    tc_commit_warp(b_drain);
    if (lane == 0) {
      mbar_drain(b_drain, 0, P.err);
      mbar_drain(b_qfull, 0, P.err);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- softmax --
    const int q = warp;                          // TMEM lane quadrant
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const bool owner = lane < 16;                // owns head row 16q + lane
    const int hl = 16 * q + (lane & 15);
    // l_run: the row sum (log-sum-exp, merge); lh_run: the sum of the weights
    // the product used (the same with the lo part; the rounded hi parts
    // without it), which normalises the output.
    float m_run = -INFINITY, l_run = 0.f, lh_run = 0.f;
    {
      // Q's dims 0..383 of head row hl into TMEM, in the M = 64 operand
      // layout (head 16q + i at lane 32q + i, dims 2c and 2c + 1 in column
      // kColQ + c): each half warp writes 32 dims of the row per store.
      const int half = lane >> 4;
      const bool have = h0 + hl < P.H;
      const uint4* const src = reinterpret_cast<const uint4*>(
          P.q + (static_cast<size_t>(r) * P.H + h0 + hl) * kLatent);
      // All of the thread's loads are in flight before the first store.
      uint4 x[kQTmemBoxes][4];
#pragma unroll
      for (int m = 0; m < kQTmemBoxes; ++m) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x[m][j] = have ? __ldg(src + (64 * m + 32 * half) / 8 + j) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int m = 0; m < kQTmemBoxes; ++m) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[4 * j] = x[m][j].x;
          v[4 * j + 1] = x[m][j].y;
          v[4 * j + 2] = x[m][j].z;
          v[4 * j + 3] = x[m][j].w;
        }
        tmem_st_16x32bx2_x16<16>(tmem + lane_base + kColQ + 32u * m, v);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(b_qtmem);
    }
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int st = t % kStages;
      const uint32_t ph = static_cast<uint32_t>((t / kStages) & 1);
      const int sb = t % kSBufs;
      ok = mbar_wait(b_sfull(sb), static_cast<uint32_t>((t / kSBufs) & 1), P.err);
      if (!ok) break;
      tc_fence_after();
      // This thread's half of its head row: keys k0 .. k0 + 23 of the tile.
      uint32_t va[16], vb[8];
      const uint32_t sa = tmem + lane_base + kColS + static_cast<uint32_t>(kT) * sb;
      tmem_ld_16x32bx2_x16<kSplitCols>(sa, va);
      tmem_ld_16x32bx2_x8<kSplitCols>(sa + 16u, vb);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(b_sempty(sb));
      // The tile's slot list was written by its gather group before kv_full.
      ok = mbar_wait(b_kvfull(st), ph, P.err);
      if (!ok) break;
      // Logits in base 2; unused slots masked.
      const int* const ti = tidx + st * kT;
      const unsigned v_lo = __ballot_sync(0xffffffffu, ti[lane] >= 0);
      const unsigned v_hi = __ballot_sync(0xffffffffu, lane < kT - 32 && ti[32 + lane] >= 0);
      const int k0 = (lane >> 4) * kSplitCols;
      const unsigned long long valid =
          ((static_cast<unsigned long long>(v_hi) << 32) | v_lo) >> k0;
      float s[kSplitCols];
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < kSplitCols; ++k) {
        const float raw_s = __uint_as_float(k < 16 ? va[k] : vb[k - 16]);
        s[k] = ((valid >> k) & 1ull) ? raw_s * P.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[k]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
      const bool raise = tmax > m_run + kRescaleLog2 || (m_run == -INFINITY && tmax > -INFINITY);
      const float m_new = raise ? tmax : m_run;
      const float alpha = raise ? exp2_fast(m_run - m_new) : 1.f;
      const float m_ref = m_new == -INFINITY ? 0.f : m_new;  // masked logits give 2^-inf = 0
      float sum = 0.f, sumh = 0.f;
      uint32_t hi[kSplitCols / 2], lo[kSplitCols / 2];
#pragma unroll
      for (int k = 0; k < kSplitCols; k += 2) {
        const float p0 = exp2_fast(s[k] - m_ref);
        const float p1 = exp2_fast(s[k + 1] - m_ref);
        sum += p0 + p1;
        const uint32_t h2 = pack2_bf16(p0, p1);
        hi[k / 2] = h2;
        const float r0 = __uint_as_float(h2 << 16), r1 = __uint_as_float(h2 & 0xFFFF0000u);
        if (use_lo) {
          lo[k / 2] = pack2_bf16(p0 - r0, p1 - r1);
        } else {
          sumh += r0 + r1;  // the weights the product uses
        }
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 16);
      sumh += __shfl_xor_sync(0xffffffffu, sumh, 16);
      l_run = l_run * alpha + sum;
      lh_run = lh_run * alpha + (use_lo ? sum : sumh);
      m_run = m_new;
      if (owner) alpha_s[hl] = alpha;
      // P buffer `pb` is free once the P.V of tile t-2 has completed.
      const int pb = t % kPStages;
      ok = mbar_wait(b_pempty(pb), static_cast<uint32_t>(((t / kPStages) & 1) ^ 1), P.err);
      if (!ok) break;
      {
        const uint32_t prow_hi = sP + (2 * pb) * kPBuf + hl * 128;
        const uint32_t prow_lo = prow_hi + kPBuf;
#pragma unroll
        for (int j = 0; j < kSplitCols / 8; ++j) {
          const int c = k0 / 8 + j;
          const uint32_t off = static_cast<uint32_t>((c ^ (hl & 7)) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow_hi + off),
                       "r"(hi[4 * j]), "r"(hi[4 * j + 1]), "r"(hi[4 * j + 2]), "r"(hi[4 * j + 3])
                       : "memory");
          if (use_lo) {
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow_lo + off),
                         "r"(lo[4 * j]), "r"(lo[4 * j + 1]), "r"(lo[4 * j + 2]), "r"(lo[4 * j + 3])
                         : "memory");
          }
        }
      }
      fence_proxy_async_smem();
      // If any head raised its running max, scale O^T (after the previous P.V).
      const bool any = named_bar_or(1, kSoftThreads, owner && raise && t > 0);
      if (any) {
        ok = mbar_wait(b_odone, static_cast<uint32_t>((t - 1) & 1), P.err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_base + kColO + 64u * blk + 32u * half;
            tmem_ld_32x32b_x32(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha_s[32 * half + j]);
            }
            tmem_st_32x32b_x32(ta, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
      }
      mbar_arrive(b_pfull(pb));
    }
    // ------------------------------------------------------------ output --
    // Per head: 1 / lh for a finished row; for a slice, lh -> l, so that the
    // merge's exact sums normalise it.
    if (owner) {
      rl_s[hl] = !(lh_run > 0.f) ? 0.f : (P.n_split > 1 ? l_run / lh_run : 1.f / lh_run);
    }
    named_bar_sync(1, kSoftThreads);
    // The MMA warp's closing commit lands once every product it issued has
    // completed (the P.V count is not enough: the product before the last
    // may still be running when the last tile's softmax ends).
    if (ok && n_tiles > 0) ok = mbar_wait(b_drain, 0, P.err);
    tc_fence_after();
    // With no tile, nothing is read from TMEM: the result is zero.
    if (ok && n_tiles == 0) ok = mbar_wait(b_qfull, 0, P.err);
    const bool good = !named_bar_or(1, kSoftThreads, !ok);
    if (good) {
      const bool split = P.n_split > 1;
      const size_t rec = split ? (static_cast<size_t>(sp) * P.Nq + r) * P.H
                               : static_cast<size_t>(r) * P.H;
      float* const dst = (split ? P.part_o : P.out) + (rec + h0) * kValue;
      // Straight from TMEM to global memory: for each head a warp writes 32
      // consecutive value dims (one 128-byte line) per store; streaming
      // stores, as nothing in this launch reads the result again.
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          const int dv = 128 * blk + 32 * q + lane;
          uint32_t o[32];
          if (n_tiles > 0) {
            tmem_ld_32x32b_x32(tmem + lane_base + kColO + 64u * blk + 32u * half, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int hh = 32 * half + j;
            float v = __uint_as_float(o[j]);
            if (!split || !use_lo) v *= rl_s[hh];
            if (h0 + hh < P.H) __stcs(dst + static_cast<size_t>(hh) * kValue + dv, v);
          }
        }
      }
      if (owner && h0 + hl < P.H) {
        if (split) {
          P.part_ml[rec + h0 + hl] = make_float2(m_run, l_run);
        } else if (P.lse) {
          P.lse[rec + h0 + hl] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}


template <bool kMasked>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t stream) {
  if (a.Nq == 0) return cudaSuccess;
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap qmap, kvmap;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kLatent),
                                static_cast<cuuint64_t>(a.Nq) * a.H};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kLatent) * 2};
    const cuuint32_t box[2] = {64, kHB};
    if (fn(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      return cudaErrorInvalidValue;
    }
  }
  kvmap = qmap;  // unused by the gather instantiation
  if (kMasked) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kLatent),
                                static_cast<cuuint64_t>(a.cache_rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kLatent) * 2};
    const cuuint32_t box[2] = {64, kT};
    if (fn(&kvmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.kv), dims,
           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = ensure_smem_limit<sparse_attn_tc_kernel<kMasked>>(kSmemTc);
  if (e != cudaSuccess) return e;
  TcParams P;
  P.q_offsets = a.q_offsets;
  P.cache = a.cache;
  P.ctx_lens = a.ctx_lens;
  P.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv);
  P.idx = a.idx;
  P.out = a.out;
  P.lse = a.lse;
  P.err = a.err;
  P.idx_prefix = a.idx_prefix ? 1 : 0;
  P.batch_ready = a.batch_ready ? 1 : 0;
  P.n_split = a.plan.n_split;
  P.split_len = a.plan.split_len;
  const size_t n_rec = static_cast<size_t>(a.plan.n_split) * a.Nq * a.H;
  P.part_o = a.part;
  P.part_ml = a.part ? reinterpret_cast<float2*>(a.part + n_rec * kValue) : nullptr;
  P.B = a.B;
  P.Nq = a.Nq;
  P.H = a.H;
  P.top_k = a.top_k;
  P.scale_log2 = a.scale * kLog2e;
  P.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    sms = 0;
  }
  P.wave = sms;  // 0: no prefetch
  const int head_blocks = (a.H + kHB - 1) / kHB;
  e = launch_pdl(sparse_attn_tc_kernel<kMasked>, dim3(a.Nq, head_blocks, a.plan.n_split),
                 dim3(kThreadsTc), static_cast<size_t>(kSmemTc), stream, 0, qmap, kvmap, P);
  if (e != cudaSuccess || a.plan.n_split == 1) return e;
  return launch_attn_merge(a, stream);
}

}  // namespace

cudaError_t launch_sparse_attn_tc(const AttnArgs& a, cudaStream_t stream) {
  return launch_tc<false>(a, stream);
}

AttnPlan masked_attn_plan(int Nq, int H, int64_t max_len, int num_sms) {
  AttnPlan p;
  p.decode = 0;
  p.tc = 1;
  p.hb = kHB;
  p.head_blocks = (H + kHB - 1) / kHB;
  // Chunks of the causal positions: about one wave of CTAs, at most
  // kMaskWords * 32 positions each, whole tiles.
  const long long base = static_cast<long long>(Nq) * p.head_blocks;
  int n = static_cast<int>(std::max<long long>(1, num_sms / std::max<long long>(1, base)));
  n = std::max(n, static_cast<int>((max_len + kMaskWords * 32 - 1) / (kMaskWords * 32)));
  n = std::min(n, 64);
  int per = static_cast<int>((max_len + n - 1) / n);
  per = (per + kT - 1) / kT * kT;
  p.split_len = std::max(per, kT);
  p.n_split = static_cast<int>((max_len + p.split_len - 1) / p.split_len);
  if (p.n_split < 1) p.n_split = 1;
  return p;
}

bool masked_attn_supported(int64_t max_len) {
  return max_len <= static_cast<int64_t>(64) * kMaskWords * 32;
}

cudaError_t launch_masked_attn(const AttnArgs& a, cudaStream_t stream) {
  return launch_tc<true>(a, stream);
}

}  // namespace dsa
