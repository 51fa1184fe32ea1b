// In-Place TTT forward and backward of the W_down fast weight on sm_100a tensor cores.
//
// Page "In-Place Test-Time Training", section "核心方法和技术细节": W_down of a gated MLP is
// the fast weight; the sequence is cut into chunks of C tokens and every chunk first applies
// the current weight, O_[i] = Z_[i] W^(i)T, then updates it with the chunk's inner-product
// gradient, W^(i+1) = W^(i) + eta Vhat_[i]^T Z_[i].
//
// The backward is the reverse-mode of that loop for J = sum_i <dO_i, O_i> + <dW_final, W_final>
// (the page gives no backward). With Wh the adjoint of the fast weight (dW_final after the last
// chunk), chunk i, from the last one down, needs
//     dVhat_i = Z_i (eta Wh_{i+1})^T,  dZ_i = dO_i W_i + Vhat_i (eta Wh_{i+1}),
//     Wh_i = Wh_{i+1} + dO_i^T Z_i     (Wh_0 is the gradient of the initial W).
//
// One launch per chunk runs every GEMM of that chunk from a shared dynamic tile queue, on
// 2-CTA clusters with tcgen05.mma.cta_group::2. A tile is 256 rows x 256 columns: each CTA of
// the pair holds 128 rows of A and 128 of the 256 columns of B in its shared memory (32 KB per
// K step of 64) and receives its 128 rows x 256 columns of the fp32 accumulator in its own
// TMEM. Tile kinds:
//   row tiles    [256 tokens x 256] = A (K-major) x B^T (K-major), A = Z_i, K = d_ff: the
//                forward's O_i (B = bf16 W_i) and the backward's dVhat_i (B = bf16 eta Wh_{i+1});
//   dz tiles     [256 tokens x 256 d_ff] = [dO_i | Vhat_i] (K-major, K = 2 d_model) x
//                [W_i ; eta Wh_{i+1}] (MN-major): the backward's dZ_i;
//   update tiles [256 d_model x 256 d_ff]: M += s X_i^T (MN-major) x Z_i (MN-major), K = C,
//                with (M, X, s) = (W, Vhat, eta) forward and (Wh, dO, 1) backward; the epilogue
//                keeps M in float32 and writes the scaled bf16 copy the next launch reads.
// Long tiles (row, then dz; the backward dz, then row) are handed out first, update tiles fill
// the remaining SMs. When a CTA takes an update tile it prefetches its float32 block of M into
// L2, so the epilogue's read-modify-write, issued after the tile's K steps, reads from L2.
// The forward and the backward are each ONE persistent launch over all chunks (over each
// document's chunks with document resets), a tile waiting (bounded) for the tiles of the
// previously processed chunk it depends on, through per-block completion counts in the
// workspace.
// Warp roles in each CTA: warp 0 issues TMA loads into a 6-stage ring, warp 1 of the leader CTA
// (rank 0) issues the pair MMAs into two TMEM accumulators of 128 x 256 fp32 per CTA, warps 2-9
// drain this CTA's accumulator rows (two warps per TMEM lane quadrant, each taking 128 of the
// 256 columns), warp 10 publishes each finished tile to the tiles of the next chunk that depend
// on it. The leader takes tiles from the queue and hands each index to its peer through
// distributed shared memory; both CTAs' loads (no multicast) complete on the leader's stage
// barrier; the MMA commits arrive on the stage and accumulator barriers of both CTAs; the peer
// signals the leader's accumulator-free and tile-free barriers remotely. Every wait is bounded.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace tttk {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, RING = 4;  // BM: rows of one CTA's half tile
constexpr int kThreads = 352;  // producer, MMA, 8 epilogue warps, completion signaller
constexpr int kEpiWarps = 8;
constexpr int kXpose = 32 * 33;  // floats of one epilogue warp's padded 32 x 32 transpose tile
constexpr uint32_t kTmemCols = 512;            // two 256-column accumulators

struct Params {
  int chunk, C, d_ff, d_model;
  int n_row_n, n_dz_n, n_upd_n;  // N tiles per 256-row block of each kind
  int n_row, n_dz, n_total;      // tiles [0, n_row) row, [n_row, n_row + n_dz) dz, rest update
  int kb_row, kb_dz, kb_dz_split, kb_upd;
  int wb_cur_row0;               // first row of the bf16 copy this launch reads
  int wb_next_row0;              // first row of the bf16 copy it writes (-1: none)
  int wc_row0;                   // first row of W_i among the saved chunk states (dz tiles)
  float acc_scale, copy_scale;   // update epilogue: M += acc_scale acc; copy = bf16(copy_scale M)
  float* M;                      // float32 matrix of the update tiles (W, or its adjoint)
  __nv_bfloat16* Mb;             // its bf16 copies
  __nv_bfloat16* Orow;           // row-tile output [T, d_model]
  __nv_bfloat16* Odz;            // dz-tile output [T, d_ff]
  int* counter;
  unsigned* err;
  // One launch over every chunk: persistent = 1 the forward (tile t belongs to chunk
  // t / tiles_per_chunk, which reads bf16 copy i (wb_saved) or i & 1 and writes the next one),
  // persistent = 2 the backward (chunk NC - 1 - t / tiles_per_chunk, reading copy i & 1 and
  // writing (i - 1) & 1, its dz tiles the saved W_i). Completion counts (kTileWarps per tile),
  // per chunk i and 256-wide block: done + UR: update tiles by row block of M; + RD: row tiles
  // by their block of M's rows; + UC: update tiles by column block (backward); + DZ: dz tiles by
  // column block (backward). A tile waits for the counts of the chunk processed before it.
  int persistent, nchunk, tiles_per_chunk, n_mblk, n_nblk, wb_saved, upd_col_major;
  int* done;
  // a persistent launch covers chunks [chunk0, chunk0 + nchunk) of the sequence (one document
  // when the sequence has document resets); chunk indices above are relative to chunk0
  int chunk0;
  // the dz tiles of a chunk are handed out before its row tiles (the backward: a dz tile needs
  // one column block of the previous chunk's adjoint copy, a row tile whole rows of it)
  int dz_first;
};

// Offsets of the completion-count arrays in Params::done.
__host__ __device__ __forceinline__ size_t done_ur(const Params& p, int i) {
  return (size_t)i * p.n_mblk;
}
__host__ __device__ __forceinline__ size_t done_rd(const Params& p, int i) {
  return ((size_t)p.nchunk + i) * p.n_mblk;
}
__host__ __device__ __forceinline__ size_t done_uc(const Params& p, int i) {
  return 2 * (size_t)p.nchunk * p.n_mblk + (size_t)i * p.n_nblk;
}
__host__ __device__ __forceinline__ size_t done_dz(const Params& p, int i) {
  return 2 * (size_t)p.nchunk * p.n_mblk + ((size_t)p.nchunk + i) * p.n_nblk;
}

constexpr int kTileWarps = 2;  // completion arrivals per pair tile (one per CTA)

// Chunk context of tile t: the chunk, its first token and the bf16 copies it reads and writes.
struct TileCtx {
  int chunk, u, row_base, wb_cur, wb_next, wc;
};
__device__ __forceinline__ TileCtx ctx_of(const Params& p, int t) {
  TileCtx c;
  c.wc = p.wc_row0;
  if (p.persistent == 2) {
    const int k = t / p.tiles_per_chunk;
    c.chunk = p.nchunk - 1 - k;
    c.u = t - k * p.tiles_per_chunk;
    c.wb_cur = (c.chunk & 1) * p.d_model;
    c.wb_next = c.chunk > 0 ? ((c.chunk - 1) & 1) * p.d_model : -1;
    c.wc = (p.chunk0 + c.chunk) * p.d_model;
  } else if (p.persistent) {
    c.chunk = t / p.tiles_per_chunk;
    c.u = t - c.chunk * p.tiles_per_chunk;
    if (p.wb_saved) {
      c.wb_cur = (p.chunk0 + c.chunk) * p.d_model;
      c.wb_next = c.chunk + 1 < p.nchunk ? (p.chunk0 + c.chunk + 1) * p.d_model : -1;
    } else {
      c.wb_cur = (c.chunk & 1) * p.d_model;
      c.wb_next = ((c.chunk + 1) & 1) * p.d_model;
    }
  } else {
    c.chunk = p.chunk;
    c.u = t;
    c.wb_cur = p.wb_cur_row0;
    c.wb_next = p.wb_next_row0;
  }
  c.row_base = (c.chunk + (p.persistent ? p.chunk0 : 0)) * p.C;
  return c;
}

__device__ __forceinline__ void red_release_add(int* a) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(a) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
// Bounded wait until *a >= target (a count other CTAs raise); false on timeout or abort.
__device__ __forceinline__ bool wait_count(const int* a, int target, const Abort& ab) {
  if (ld_acquire_gpu(a) >= target) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(128);
    if (ld_acquire_gpu(a) >= target) return true;
    if ((it & 15u) == 0) {
      if (*ab.flag) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *ab.flag = 1;
        atomicOr(ab.err, ERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

enum Kind { KIND_ROW = 0, KIND_DZ = 1, KIND_UPD = 2 };

constexpr int MBOX = 64;  // float32 columns of M per L2 prefetch box (box: 128 rows x 64)

// Prefetch of one box of a 2-D tensor map into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(c0), "r"(c1)
               : "memory");
}

struct Tile {
  int kind, m0, n0, nkb;
};

// Tile t of a launch whose tiles are TM rows high (256: a CTA pair).
template <int TM>
__device__ __forceinline__ Tile decode(const Params& p, int t) {
  Tile x;
  if (p.dz_first) t = t < p.n_dz ? t + p.n_row : t < p.n_dz + p.n_row ? t - p.n_dz : t;
  if (t < p.n_row) {
    x.kind = KIND_ROW;
    x.m0 = (t / p.n_row_n) * TM;  // token offset inside the chunk
    x.n0 = (t % p.n_row_n) * BN;  // d_model column
    x.nkb = p.kb_row;
  } else if (t < p.n_row + p.n_dz) {
    const int u = t - p.n_row;
    x.kind = KIND_DZ;
    if (p.dz_first) {
      // column blocks in the order the previous chunk's (column-major) update tiles finish them
      const int n_tok = p.n_dz / p.n_dz_n;
      x.m0 = (u % n_tok) * TM;
      x.n0 = (u / n_tok) * BN;
    } else {
      x.m0 = (u / p.n_dz_n) * TM;   // token offset inside the chunk
      x.n0 = (u % p.n_dz_n) * BN;   // d_ff column
    }
    x.nkb = p.kb_dz;
  } else {
    const int u = t - p.n_row - p.n_dz;
    x.kind = KIND_UPD;
    if (p.upd_col_major) {
      // the backward: the column blocks of the adjoint copy complete one after another, which
      // is the order the next chunk's dz tiles need them in
      const int n_m = (p.d_model + TM - 1) / TM;
      x.m0 = (u % n_m) * TM;
      x.n0 = (u / n_m) * BN;
    } else {
      x.m0 = (u / p.n_upd_n) * TM;  // d_model row
      x.n0 = (u % p.n_upd_n) * BN;  // d_ff column
    }
    x.nkb = p.kb_upd;
  }
  return x;
}


// ============================================================================= CTA pairs
constexpr int PTM = 2 * BM;                     // rows of a pair tile
constexpr int P_STAGES = 6;
constexpr uint32_t PA_BYTES = BM * BK * 2;      // 16 KB: this CTA's 128 rows of A
constexpr uint32_t PB_BYTES = (BN / 2) * BK * 2;  // 16 KB: this CTA's 128 columns of B
constexpr uint32_t P_STAGE = PA_BYTES + PB_BYTES;
constexpr int kPairTileReaders = 2 * (2 + kEpiWarps);  // leader MMA, peer producer, and in each
                                                       // CTA the epilogue and the signaller

struct __align__(8) PairBars {
  uint64_t full[P_STAGES], empty[P_STAGES], acc_full[2], acc_empty[2], tile_full[RING],
      tile_empty[RING], tile_done[2];
  int ring[RING];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kPairSmemBytes =
    P_STAGES * P_STAGE + sizeof(PairBars) + kEpiWarps * kXpose * sizeof(float) + 1024;
static_assert(kPairSmemBytes <= 232448, "shared memory of one CTA");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory word in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// Arrive (release at cluster scope) on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with acquire at cluster scope (for what the other CTA of the pair wrote).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, const Abort& ab) {
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*ab.flag) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *ab.flag = 1;
        atomicOr(ab.err, ERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}
// 2-D TMA load into this CTA's shared memory whose completion counts on `bar_cluster`, an
// mbarrier of either CTA of the pair (here always the leader's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the mbarrier at this shared-memory offset in both CTAs of the pair when
// every pair MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(both)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    inplace_pair_kernel(const __grid_constant__ CUtensorMap tm_za,    // Z, K-major, 128 rows
                        const __grid_constant__ CUtensorMap tm_zb,    // Z, MN-major boxes
                        const __grid_constant__ CUtensorMap tm_mb,    // bf16 copy, K-major, 128 rows
                        const __grid_constant__ CUtensorMap tm_x,     // Vhat or dO, MN-major
                        const __grid_constant__ CUtensorMap tm_do,    // dO, K-major
                        const __grid_constant__ CUtensorMap tm_vk,    // Vhat, K-major
                        const __grid_constant__ CUtensorMap tm_wc,    // saved W_i, MN-major
                        const __grid_constant__ CUtensorMap tm_mbn,   // bf16 copy, MN-major
                        const __grid_constant__ CUtensorMap tm_mf,    // float32 M (prefetch)
                        const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  PairBars* bars = reinterpret_cast<PairBars*>(smem + P_STAGES * P_STAGE);
  float* xpose = reinterpret_cast<float*>(smem + P_STAGES * P_STAGE + sizeof(PairBars));
  const uint32_t stage0 = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int half = (int)rank * BM;  // this CTA's first row (and first B column) of a pair tile
  Abort ab{&bars->abort_flag, p.err};
#define PB(x) smem_u32(&bars->x)

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(PB(full[s]), 1);
      mbar_init(PB(empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(PB(acc_full[a]), 1);
      mbar_init(PB(acc_empty[a]), 2 * kEpiWarps);
      mbar_init(PB(tile_done[a]), kEpiWarps);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(PB(tile_full[r]), 1);
      mbar_init(PB(tile_empty[r]), kPairTileReaders);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_za);
    tma_prefetch_desc(&tm_zb);
    tma_prefetch_desc(&tm_mb);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_mf);
    if (p.n_dz) {
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_vk);
      tma_prefetch_desc(&tm_wc);
      tma_prefetch_desc(&tm_mbn);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(PB(tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int r = 0, s = 0;
      uint32_t rph = 0, sph = 0;
      for (;;) {
        int t;
        if (leader) {
          if (!mbar_wait_cluster(PB(tile_empty[r]), rph ^ 1, ab)) break;
          t = atomicAdd(p.counter, 1);
          bars->ring[r] = t;
          st_cluster_u32(peer_addr(PB(ring[r]), 1), t);
          mbar_arrive(PB(tile_full[r]));
          mbar_arrive_cluster(peer_addr(PB(tile_full[r]), 1));
        } else {
          if (!mbar_wait_cluster(PB(tile_full[r]), rph, ab)) break;
          t = bars->ring[r];
          mbar_arrive_cluster(peer_addr(PB(tile_empty[r]), 0));
        }
        if (++r == RING) { r = 0; rph ^= 1; }
        if (t >= p.n_total) break;
        const TileCtx cx = ctx_of(p, t);
        const Tile x = decode<PTM>(p, cx.u);
        const int row_base = cx.row_base;
        const int m0 = x.m0 + half, nb = x.n0 + half;  // this CTA's rows of A, columns of B
        bool ok = true;
        // the chunk processed just before this one (forward: i - 1, backward: i + 1)
        const int prev = p.persistent == 2 ? cx.chunk + 1 : cx.chunk - 1;
        if (p.persistent && prev >= 0 && prev < p.nchunk) {
          const int n_tok = p.n_row / p.n_row_n;        // row (and dz) tiles per column block
          const int n_m = (p.d_model + PTM - 1) / PTM;  // update tiles per column block
          const int* d = p.done;
          if (p.persistent == 1) {
            // forward: a row tile reads the bf16 rows [n0, n0 + 256) of W that the previous
            // chunk's update tiles wrote; an update tile rewrites rows [m0, m0 + 256) of W after
            // the previous chunk's update tiles, and of the bf16 copy the previous chunk's row
            // tiles read (the copies rotate)
            if (x.kind == KIND_ROW)
              ok = wait_count(d + done_ur(p, prev) + x.n0 / PTM, kTileWarps * p.n_upd_n, ab);
            else
              ok = wait_count(d + done_ur(p, prev) + x.m0 / PTM, kTileWarps * p.n_upd_n, ab) &&
                   wait_count(d + done_rd(p, prev) + x.m0 / PTM, kTileWarps * n_tok, ab);
          } else {
            // backward: a row tile reads rows [n0, n0 + 256) of the adjoint copy, a dz tile
            // every row of its columns [n0, n0 + 256), both written by the previous chunk's
            // update tiles; an update tile rewrites its block of the adjoint after the previous
            // chunk's update tiles of those rows, and of the copy the previous chunk's row tiles
            // (its rows) and dz tiles (its columns) read
            if (x.kind == KIND_ROW)
              ok = wait_count(d + done_ur(p, prev) + x.n0 / PTM, kTileWarps * p.n_upd_n, ab);
            else if (x.kind == KIND_DZ)
              ok = wait_count(d + done_uc(p, prev) + x.n0 / BN, kTileWarps * n_m, ab);
            else
              ok = wait_count(d + done_ur(p, prev) + x.m0 / PTM, kTileWarps * p.n_upd_n, ab) &&
                   wait_count(d + done_rd(p, prev) + x.m0 / PTM, kTileWarps * n_tok, ab) &&
                   wait_count(d + done_dz(p, prev) + x.n0 / BN, kTileWarps * n_tok, ab);
          }
          // what those tiles stored (generic proxy) is read next by TMA (async proxy)
          asm volatile("fence.proxy.async.global;" ::: "memory");
          if (!ok) break;
        }
        if (x.kind == KIND_UPD && m0 < p.d_model)
          for (int j = 0; j < BN / MBOX; ++j) tma_prefetch_l2_2d(&tm_mf, x.n0 + MBOX * j, m0);
        for (int kb = 0; kb < x.nkb && ok; ++kb) {
          if (!mbar_wait(PB(empty[s]), sph ^ 1, ab)) { ok = false; break; }
          // both halves of the stage complete on the leader's barrier
          if (leader) mbar_arrive_expect_tx(PB(full[s]), 2 * P_STAGE);
          const uint32_t fb = peer_addr(PB(full[s]), 0);
          const uint32_t sa = stage0 + s * P_STAGE, sb = sa + PA_BYTES;
          if (x.kind == KIND_ROW) {
            tma_load_2d_pair(sa, &tm_za, fb, kb * BK, row_base + m0);
            tma_load_2d_pair(sb, &tm_mb, fb, kb * BK, cx.wb_cur + nb);
          } else if (x.kind == KIND_DZ) {
            // K runs over [dO_i | Vhat_i] against [W_i ; eta Wh_{i+1}]
            const bool first = kb < p.kb_dz_split;
            const int k0 = (first ? kb : kb - p.kb_dz_split) * BK;
            tma_load_2d_pair(sa, first ? &tm_do : &tm_vk, fb, k0, row_base + m0);
            const CUtensorMap* mb = first ? &tm_wc : &tm_mbn;
            const int r0 = (first ? cx.wc : cx.wb_cur) + k0;
            for (int j = 0; j < 2; ++j) tma_load_2d_pair(sb + 8192 * j, mb, fb, nb + 64 * j, r0);
          } else {
            const int tok = row_base + kb * BK;
            tma_load_2d_pair(sa, &tm_x, fb, m0, tok);
            tma_load_2d_pair(sa + 8192, &tm_x, fb, m0 + 64, tok);
            for (int j = 0; j < 2; ++j) tma_load_2d_pair(sb + 8192 * j, &tm_zb, fb, nb + 64 * j, tok);
          }
          if (++s == P_STAGES) { s = 0; sph ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issue (the leader's thread)
    if (lane == 0 && leader) {
      int r = 0, s = 0, acc = 0;
      uint32_t rph = 0, sph = 0, aph = 0;
      const uint32_t id_row = idesc_bf16(PTM, BN, 0, 0);
      const uint32_t id_dz = idesc_bf16(PTM, BN, 0, 1);
      const uint32_t id_upd = idesc_bf16(PTM, BN, 1, 1);
      for (;;) {
        if (!mbar_wait(PB(tile_full[r]), rph, ab)) break;
        const int t = bars->ring[r];
        mbar_arrive(PB(tile_empty[r]));
        if (++r == RING) { r = 0; rph ^= 1; }
        if (t >= p.n_total) break;
        const Tile x = decode<PTM>(p, ctx_of(p, t).u);
        // both CTAs' epilogues have drained this accumulator
        if (!mbar_wait_cluster(PB(acc_empty[acc]), aph ^ 1, ab)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        const uint32_t id = x.kind == KIND_ROW ? id_row : x.kind == KIND_DZ ? id_dz : id_upd;
        const bool a_kmaj = x.kind != KIND_UPD, b_kmaj = x.kind == KIND_ROW;
        bool ok = true;
        for (int kb = 0; kb < x.nkb; ++kb) {
          if (!mbar_wait(PB(full[s]), sph, ab)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = stage0 + s * P_STAGE, sb = sa + PA_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = a_kmaj ? sdesc_sw128(sa + kk * 32, 16, 1024)
                                       : sdesc_sw128(sa + kk * 2048, 8192, 1024);
            const uint64_t bd = b_kmaj ? sdesc_sw128(sb + kk * 32, 16, 1024)
                                       : sdesc_sw128(sb + kk * 2048, 8192, 1024);
            mma_bf16_pair(d, ad, bd, id, (kb | kk) != 0);
          }
          mma_commit_pair(PB(empty[s]));  // the stage is free in both CTAs
          if (++s == P_STAGES) { s = 0; sph ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(PB(acc_full[acc]));
        if (++acc == 2) { acc = 0; aph ^= 1; }
      }
    }
  } else if (warp == 2 + kEpiWarps) {
    // ------------------------------------------ completion signaller (both CTAs, one thread)
    // After the eight epilogue warps of this CTA have stored a tile (tile_done), raise the
    // tile's completion count with release semantics at GPU scope; the epilogue warps never wait
    // for their stores to become visible.
    if (lane == 0) {
      int r = 0, acc = 0;
      uint32_t rph = 0, aph = 0;
      for (;;) {
        if (!mbar_wait_cluster(PB(tile_full[r]), rph, ab)) break;
        const int t = bars->ring[r];
        if (leader)
          mbar_arrive(PB(tile_empty[r]));
        else
          mbar_arrive_cluster(peer_addr(PB(tile_empty[r]), 0));
        if (++r == RING) { r = 0; rph ^= 1; }
        if (t >= p.n_total) break;
        const TileCtx cx = ctx_of(p, t);
        const Tile x = decode<PTM>(p, cx.u);
        if (!mbar_wait(PB(tile_done[acc]), aph, ab)) break;
        if (p.persistent) {
          int* d = p.done;
          if (x.kind == KIND_UPD) {
            red_release_add(d + done_ur(p, cx.chunk) + x.m0 / PTM);
            if (p.persistent == 2) red_release_add(d + done_uc(p, cx.chunk) + x.n0 / BN);
          } else if (x.kind == KIND_ROW) {
            red_release_add(d + done_rd(p, cx.chunk) + x.n0 / PTM);
          } else {
            red_release_add(d + done_dz(p, cx.chunk) + x.n0 / BN);
          }
        }
        if (++acc == 2) { acc = 0; aph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    // Warp w drains TMEM lanes 32*(w%4) .. +31 (thread = one row of this CTA's half) and
    // columns [128 h, 128 h + 128) with h = (w - 2) / 4, as in the single-CTA kernel.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int hcol = (warp - 2) / 4;
    int r = 0, acc = 0;
    uint32_t rph = 0, aph = 0;
    for (;;) {
      if (!mbar_wait_cluster(PB(tile_full[r]), rph, ab)) break;
      const int t = bars->ring[r];
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(PB(tile_empty[r]));
        else
          mbar_arrive_cluster(peer_addr(PB(tile_empty[r]), 0));
      }
      if (++r == RING) { r = 0; rph ^= 1; }
      if (t >= p.n_total) break;
      const TileCtx cx = ctx_of(p, t);
      const Tile x = decode<PTM>(p, cx.u);
      const int row_base = cx.row_base;
      const int m0 = x.m0 + half;
      if (!mbar_wait(PB(acc_full[acc]), aph, ab)) break;
      __syncwarp();
      tc_fence_after();
      const int cb0 = hcol * (BN / 64), cb1 = cb0 + BN / 64;
      if (x.kind != KIND_UPD) {
        // bf16 rows of O_i / dVhat_i ([T, d_model]) or dZ_i ([T, d_ff]); rows past the chunk
        // (a pair tile reaching beyond C) are not written
        const int ncol = x.kind == KIND_ROW ? p.d_model : p.d_ff;
        const bool row_ok = m0 + row < p.C;
        __nv_bfloat16* out = (x.kind == KIND_ROW ? p.Orow : p.Odz) +
                             (size_t)(row_base + (row_ok ? m0 + row : 0)) * ncol;
        for (int cb = cb0; cb < cb1; ++cb) {
          float v[32];
          tmem_ld32(tmem_addr(tmem, q * 32, acc * BN + cb * 32), v);
          tmem_wait_ld();
          const int col0 = x.n0 + cb * 32;
          if (row_ok && col0 < ncol) {
            uint4* dst = reinterpret_cast<uint4*>(out + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                  pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                  pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
        }
      } else {
        // fp32 read-modify-write of M and its scaled bf16 copy, as in the single-CTA kernel;
        // a warp whose 32 rows lie past d_model (the upper half of the last pair tile when
        // d_model is not a multiple of 256) touches no memory
        float* xt = xpose + (warp - 2) * kXpose;
        const int mbase = m0 + q * 32;
        const bool rows_ok = mbase < p.d_model;  // d_model is a multiple of 128
        const float s = p.acc_scale, cs = p.copy_scale;
        const size_t ld = p.d_ff;
        auto valid = [&](int cb) { return rows_ok && x.n0 + cb * 32 < p.d_ff; };
        auto load_block = [&](int cb, float (&w)[32]) {
          const float* lp = p.M + (size_t)mbase * ld + x.n0 + cb * 32 + lane;
#pragma unroll
          for (int rr = 0; rr < 32; ++rr, lp += ld) w[rr] = __ldcg(lp);
        };
        auto stage_acc = [&](int cb) {
          float v[32];
          tmem_ld32(tmem_addr(tmem, q * 32, acc * BN + cb * 32), v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) xt[lane * 33 + j] = v[j];
          __syncwarp();
        };
        auto store_block = [&](int cb, const float (&w)[32]) {
          const int col = x.n0 + cb * 32 + lane;
          float* mp = p.M + (size_t)mbase * ld + col;
          __nv_bfloat16* bp =
              cx.wb_next >= 0 ? p.Mb + (size_t)(cx.wb_next + mbase) * ld + col : nullptr;
#pragma unroll
          for (int rr = 0; rr < 32; ++rr, mp += ld) {
            const float o = w[rr] + s * xt[rr * 33 + lane];
            *mp = o;
            if (bp) {
              *bp = __float2bfloat16_rn(cs * o);
              bp += ld;
            }
          }
        };
        float wa[32], wb[32];
        if (valid(cb0)) load_block(cb0, wa);
#pragma unroll
        for (int i = 0; i < BN / 64; i += 2) {
          const int cb = cb0 + i;
          stage_acc(cb);
          if (valid(cb + 1)) load_block(cb + 1, wb);
          if (valid(cb)) store_block(cb, wa);
          __syncwarp();
          stage_acc(cb + 1);
          if (i + 2 < BN / 64 && valid(cb + 2)) load_block(cb + 2, wa);
          if (valid(cb + 1)) store_block(cb + 1, wb);
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(PB(acc_empty[acc]));
        else
          mbar_arrive_cluster(peer_addr(PB(acc_empty[acc]), 0));
        // this warp's stores of the tile (the whole warp's, ordered before this thread's by the
        // __syncwarp) are done: the signaller publishes them with the tile's completion count
        mbar_arrive(PB(tile_done[acc]));
      }
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no MMA of the leader still writes the peer's TMEM
  if (bars->abort_flag) __nanosleep(100000);  // let any load issued before the abort land
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
#undef PB
}

// dst = bf16(scale * src) over n elements.
__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               size_t n, float scale) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(scale * src[i]);
}


// dst += src over n floats (n a multiple of 4).
__global__ void add_kernel(float* __restrict__ dst, const float* __restrict__ src, size_t n4) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<float4*>(dst)[i];
    const float4 b = reinterpret_cast<const float4*>(src)[i];
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    reinterpret_cast<float4*>(dst)[i] = a;
  }
}

// Depthwise convolution over the current and the next k - 1 tokens, zero past the last one:
// Y[t, c] = sum_{j<k} w[j, c] X0[t + j, c]. One thread per 8 channels and a run of tokens;
// a warp's loads of one token row are contiguous.
constexpr int kMaxTaps = 8;
__global__ void __launch_bounds__(128)
    conv_future_kernel(const __nv_bfloat16* __restrict__ X0, const float* __restrict__ w,
                       __nv_bfloat16* __restrict__ Y, int T, int d, int k, int run) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;  // group of 8 channels
  if (c8 * 8 >= d) return;
  float wv[kMaxTaps][8];
#pragma unroll
  for (int j = 0; j < kMaxTaps; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) wv[j][e] = j < k ? w[(size_t)j * d + c8 * 8 + e] : 0.f;
  const int t0 = blockIdx.y * run, t1 = min(T, t0 + run);
  for (int t = t0; t < t1; ++t) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
      if (j >= k || t + j >= T) break;
      const uint4 x = *reinterpret_cast<const uint4*>(X0 + (size_t)(t + j) * d + c8 * 8);
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        acc[2 * h] += wv[j][2 * h] * bf16lo(xw[h]);
        acc[2 * h + 1] += wv[j][2 * h + 1] * bf16hi(xw[h]);
      }
    }
    *reinterpret_cast<uint4*>(Y + (size_t)t * d + c8 * 8) =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

// Transposed convolution and the tap gradients of one run of tokens, 8 channels per thread:
// dX0[t, c] = sum_{j<k, t-j>=0} w[j, c] dY[t-j, c]; part[run, j, c] = sum_{t in run, t+j<T}
// dY[t, c] X0[t+j, c] (summed over the runs by conv_taps_reduce2_kernel).
__global__ void __launch_bounds__(128)
    conv_future_bwd_kernel(const __nv_bfloat16* __restrict__ X0, const float* __restrict__ w,
                           const __nv_bfloat16* __restrict__ dY, __nv_bfloat16* __restrict__ dX0,
                           float* __restrict__ part, int T, int d, int k, int run) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
  if (c8 * 8 >= d) return;
  float wv[kMaxTaps][8], pw[kMaxTaps][8];
#pragma unroll
  for (int j = 0; j < kMaxTaps; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      wv[j][e] = j < k ? w[(size_t)j * d + c8 * 8 + e] : 0.f;
      pw[j][e] = 0.f;
    }
  const int t0 = blockIdx.y * run, t1 = min(T, t0 + run);
  auto load8 = [&](const __nv_bfloat16* base, int t, float (&v)[8]) {
    const uint4 x = *reinterpret_cast<const uint4*>(base + (size_t)t * d + c8 * 8);
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = bf16lo(xw[h]);
      v[2 * h + 1] = bf16hi(xw[h]);
    }
  };
  for (int t = t0; t < t1; ++t) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, g[8], x[8];
    load8(dY, t, g);
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
      if (j >= k) break;
      if (t - j >= 0) {
        float gj[8];
        load8(dY, t - j, gj);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += wv[j][e] * gj[e];
      }
      if (t + j < T) {
        load8(X0, t + j, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) pw[j][e] += g[e] * x[e];
      }
    }
    *reinterpret_cast<uint4*>(dX0 + (size_t)t * d + c8 * 8) =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
#pragma unroll
  for (int j = 0; j < kMaxTaps; ++j)
    if (j < k)
#pragma unroll
      for (int e = 0; e < 8; ++e) part[((size_t)blockIdx.y * k + j) * d + c8 * 8 + e] = pw[j][e];
}

// Faster forms of the two convolutions for k <= 4 taps (the NTP workload uses 4): each
// thread slides a window of token rows through registers, so every row of X0 (and of dY) is
// loaded once per run instead of k times, and four rows are loaded together ahead of their
// use. Runs are 64 tokens; 64 threads (8 channels each) cover 512 channels per block.
constexpr int kRun = 64;

__device__ __forceinline__ uint4 ld_row8(const __nv_bfloat16* base, int t, int T, int d, int c8) {
  return t < T && t >= 0 ? __ldg(reinterpret_cast<const uint4*>(base + (size_t)t * d + c8 * 8))
                         : make_uint4(0u, 0u, 0u, 0u);
}
__device__ __forceinline__ void unpack8(const uint4& x, float (&v)[8]) {
  const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = bf16lo(xw[h]);
    v[2 * h + 1] = bf16hi(xw[h]);
  }
}

template <int K>
__global__ void __launch_bounds__(64)
    conv_future_win_kernel(const __nv_bfloat16* __restrict__ X0, const float* __restrict__ w,
                           __nv_bfloat16* __restrict__ Y, int T, int d) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
  if (c8 * 8 >= d) return;
  float wv[K][8];
#pragma unroll
  for (int j = 0; j < K; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) wv[j][e] = w[(size_t)j * d + c8 * 8 + e];
  const int t0 = blockIdx.y * kRun;
  // rows t .. t + K - 1 of X0 for the next output token t
  uint4 win[K + 3];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) win[j] = ld_row8(X0, t0 + j, T, d, c8);
#pragma unroll 1
  for (int t = t0; t < t0 + kRun; t += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) win[K - 1 + u] = ld_row8(X0, t + K - 1 + u, T, d, c8);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < K; ++j) {
        float x[8];
        unpack8(win[u + j], x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += wv[j][e] * x[e];
      }
      *reinterpret_cast<uint4*>(Y + (size_t)(t + u) * d + c8 * 8) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
#pragma unroll
    for (int j = 0; j < K - 1; ++j) win[j] = win[j + 4];
  }
}

// dX0[t] = sum_j w[j] dY[t - j] (a window of past dY rows) and the run's tap partials
// part[run, j] = sum_t dY[t] X0[t + j] (a window of future X0 rows).
template <int K>
__global__ void __launch_bounds__(64)
    conv_future_bwd_win_kernel(const __nv_bfloat16* __restrict__ X0, const float* __restrict__ w,
                               const __nv_bfloat16* __restrict__ dY, __nv_bfloat16* __restrict__ dX0,
                               float* __restrict__ part, int T, int d) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
  if (c8 * 8 >= d) return;
  float wv[K][8], pw[K][8];
#pragma unroll
  for (int j = 0; j < K; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      wv[j][e] = w[(size_t)j * d + c8 * 8 + e];
      pw[j][e] = 0.f;
    }
  const int t0 = blockIdx.y * kRun;
  uint4 gw[K + 3];  // dY rows t - K + 1 .. t (+3)
  uint4 xw[K + 3];  // X0 rows t .. t + K - 1 (+3)
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    gw[j] = ld_row8(dY, t0 - K + 1 + j, T, d, c8);
    xw[j] = ld_row8(X0, t0 + j, T, d, c8);
  }
#pragma unroll 1
  for (int t = t0; t < t0 + kRun; t += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      gw[K - 1 + u] = ld_row8(dY, t + u, T, d, c8);
      xw[K - 1 + u] = ld_row8(X0, t + K - 1 + u, T, d, c8);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, g[8];
      unpack8(gw[K - 1 + u], g);
#pragma unroll
      for (int j = 0; j < K; ++j) {
        float y[8], x[8];
        unpack8(gw[K - 1 + u - j], y);  // dY[t + u - j]
        unpack8(xw[u + j], x);          // X0[t + u + j]
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[e] += wv[j][e] * y[e];
          pw[j][e] += g[e] * x[e];
        }
      }
      *reinterpret_cast<uint4*>(dX0 + (size_t)(t + u) * d + c8 * 8) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
      gw[j] = gw[j + 4];
      xw[j] = xw[j + 4];
    }
  }
#pragma unroll
  for (int j = 0; j < K; ++j) {
    float4* dst = reinterpret_cast<float4*>(part + ((size_t)blockIdx.y * K + j) * d + c8 * 8);
    dst[0] = make_float4(pw[j][0], pw[j][1], pw[j][2], pw[j][3]);
    dst[1] = make_float4(pw[j][4], pw[j][5], pw[j][6], pw[j][7]);
  }
}

// dconv_w[i] = sum over the runs of part[run, i], i over k d: 32 consecutive i per block, the
// runs split over 8 thread rows that each add theirs in order, then the 8 row sums in order
// (the result does not depend on scheduling).
__global__ void __launch_bounds__(256)
    conv_taps_reduce2_kernel(const float* __restrict__ part, float* __restrict__ dw, int nrun, int kd) {
  __shared__ float red[8][33];
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int i = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (i < kd)
    for (int r = g; r < nrun; r += 8) s += part[(size_t)r * kd + i];
  red[g][lane] = s;
  __syncthreads();
  if (g == 0 && i < kd) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][lane];
    dw[i] = t;
  }
}

// Launch helpers: the windowed kernels for k <= 4, the per-token kernels otherwise.
cudaError_t conv_fwd_launch(const __nv_bfloat16* X0, const float* w, __nv_bfloat16* Y, int T,
                            int d, int k, cudaStream_t s) {
  const dim3 g((d / 8 + 63) / 64, T / kRun);
  switch (k) {
    case 1: conv_future_win_kernel<1><<<g, 64, 0, s>>>(X0, w, Y, T, d); break;
    case 2: conv_future_win_kernel<2><<<g, 64, 0, s>>>(X0, w, Y, T, d); break;
    case 3: conv_future_win_kernel<3><<<g, 64, 0, s>>>(X0, w, Y, T, d); break;
    case 4: conv_future_win_kernel<4><<<g, 64, 0, s>>>(X0, w, Y, T, d); break;
    default:
      conv_future_kernel<<<dim3((d / 8 + 127) / 128, T / kRun), 128, 0, s>>>(X0, w, Y, T, d, k, kRun);
  }
  return cudaGetLastError();
}
cudaError_t conv_bwd_launch(const __nv_bfloat16* X0, const float* w, const __nv_bfloat16* dY,
                            __nv_bfloat16* dX0, float* part, float* dw, int T, int d, int k,
                            cudaStream_t s) {
  const int nrun = T / kRun;
  const dim3 g((d / 8 + 63) / 64, nrun);
  switch (k) {
    case 1: conv_future_bwd_win_kernel<1><<<g, 64, 0, s>>>(X0, w, dY, dX0, part, T, d); break;
    case 2: conv_future_bwd_win_kernel<2><<<g, 64, 0, s>>>(X0, w, dY, dX0, part, T, d); break;
    case 3: conv_future_bwd_win_kernel<3><<<g, 64, 0, s>>>(X0, w, dY, dX0, part, T, d); break;
    case 4: conv_future_bwd_win_kernel<4><<<g, 64, 0, s>>>(X0, w, dY, dX0, part, T, d); break;
    default:
      conv_future_bwd_kernel<<<dim3((d / 8 + 127) / 128, nrun), 128, 0, s>>>(X0, w, dY, dX0, part,
                                                                            T, d, k, kRun);
  }
  conv_taps_reduce2_kernel<<<(k * d + 31) / 32, 256, 0, s>>>(part, dw, nrun, k * d);
  return cudaGetLastError();
}

struct Launch {
  int sms;
  int pairs;  // CTA pairs that fit on the device at once
};

cudaError_t prepare(Launch* l) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&l->sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(inplace_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kPairSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (l->sms / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, inplace_pair_kernel, &cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = l->sms / 2;
  }
  l->pairs = n;
  return cudaSuccess;
}

// Tile counts of a pair launch: row and dz tiles over `rows` token rows, update tiles over the
// d_model rows of M, each 256 rows high (the N counts are set by the caller).
void pair_tiles(Params& p, int row_rows, int dz_rows, int upd_rows) {
  auto blocks = [](int rows) { return (rows + PTM - 1) / PTM; };
  p.n_row = row_rows ? blocks(row_rows) * p.n_row_n : 0;
  p.n_dz = dz_rows ? blocks(dz_rows) * p.n_dz_n : 0;
  p.n_total = p.n_row + p.n_dz + (upd_rows ? blocks(upd_rows) * p.n_upd_n : 0);
}

// One launch of the tile program on CTA pairs (grid: the co-resident pairs, at most one per
// tile).
void launch_pairs(const Launch& l, const Params& p, cudaStream_t s, const CUtensorMap& za,
                  const CUtensorMap& zb, const CUtensorMap& mb, const CUtensorMap& x,
                  const CUtensorMap& dO, const CUtensorMap& vk, const CUtensorMap& wc,
                  const CUtensorMap& mbn, const CUtensorMap& mf) {
  const int pairs = p.n_total < l.pairs ? p.n_total : l.pairs;
  inplace_pair_kernel<<<2 * pairs, kThreads, kPairSmemBytes, s>>>(za, zb, mb, x, dO, vk, wc, mbn,
                                                                  mf, p);
}

}  // namespace

// Two bf16 copies of a d_model x d_ff matrix (read by one chunk, written for the next), then
// one tile counter per chunk and the persistent launches' completion counts (two per chunk and
// 256 rows of the matrix, two per chunk and 256 of its columns); with document resets one
// float32 d_model x d_ff matrix more (the initial W forward, the running adjoint backward).
size_t inplace_workspace(int T, int d_ff, int d_model, int C, bool docs) {
  const size_t wb = 2 * (size_t)d_model * d_ff * 2;
  const size_t nc = (size_t)(T / C), n_mblk = ((size_t)d_model + PTM - 1) / PTM,
               n_nblk = ((size_t)d_ff + BN - 1) / BN;
  const size_t counters = ((nc + 2 * nc * (n_mblk + n_nblk)) * sizeof(int) + 255) & ~size_t(255);
  return wb + counters + (docs ? (size_t)d_model * d_ff * 4 : 0);
}

cudaError_t inplace_run(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                        const void* Vhat, float* W, void* O, void* W_chunks, const bool* reset,
                        void* ws, unsigned* err, cudaStream_t s) {
  const int NC = T / C;
  const size_t nW = (size_t)d_model * d_ff;
  // bf16 W_i: the caller's [NC, d_model, d_ff] chunk states when given, else two rotating copies
  __nv_bfloat16* Wb = W_chunks ? static_cast<__nv_bfloat16*>(W_chunks)
                               : static_cast<__nv_bfloat16*>(ws);
  const size_t wb_rows = W_chunks ? (size_t)NC * d_model : 2 * (size_t)d_model;
  int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 2 * (size_t)d_model * d_ff * 2);
  // with document resets: the initial W, kept after the counters
  float* W0 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) +
                                       inplace_workspace(T, d_ff, d_model, C, false));
  CUtensorMap tza, tzb, twb, tvh, tmf;
  if (!make_tmap_bf16(&tza, Z, d_ff, T, d_ff, BK, BM) ||
      !make_tmap_bf16(&tzb, Z, d_ff, T, d_ff, 64, BK) ||
      !make_tmap_bf16(&twb, Wb, d_ff, wb_rows, d_ff, BK, BN / 2) ||
      !make_tmap_bf16(&tvh, Vhat, d_model, T, d_model, 64, BK) ||
      !make_tmap_f32(&tmf, W, d_ff, d_model, d_ff, MBOX, BM))
    return cudaErrorInvalidValue;
  Launch l;
  cudaError_t e = prepare(&l);
  if (e != cudaSuccess) return e;
  if (reset && (e = cudaMemcpyAsync(W0, W, nW * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return e;
  const int n_mblk = (d_model + PTM - 1) / PTM, n_nblk = (d_ff + BN - 1) / BN;
  const size_t n_counters = ((size_t)NC + 2 * (size_t)NC * (n_mblk + n_nblk)) * sizeof(int);
  Params p{};
  p.C = C;
  p.d_ff = d_ff;
  p.d_model = d_model;
  p.n_row_n = (d_model + BN - 1) / BN;
  p.n_upd_n = (d_ff + BN - 1) / BN;
  pair_tiles(p, C, 0, d_model);
  p.kb_row = d_ff / BK;
  p.kb_upd = C / BK;
  p.acc_scale = lr;
  p.copy_scale = 1.f;
  p.M = W;
  p.Mb = Wb;
  p.Orow = static_cast<__nv_bfloat16*>(O);
  p.err = err;
  // One persistent launch per document (the whole sequence without resets): each tile waits for
  // the tiles of the document's previous chunk it depends on. A document after the first starts
  // from the initial W, kept in the workspace.
  p.persistent = 1;
  p.n_mblk = n_mblk;
  p.n_nblk = n_nblk;
  p.wb_saved = W_chunks != nullptr;
  p.done = counters + NC;
  p.counter = counters;
  const int per_chunk = p.n_total;
  int launches = 0;
  for (int a = 0; a < NC;) {
    int b = a + 1;
    while (b < NC && !(reset && reset[b])) ++b;
    if (a > 0 && (e = cudaMemcpyAsync(W, W0, nW * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
      return e;
    // the bf16 copy the document's first chunk applies
    to_bf16_kernel<<<l.sms * 4, 256, 0, s>>>(a > 0 ? W0 : W,
                                             Wb + (W_chunks ? (size_t)a * d_model * d_ff : 0),
                                             nW, 1.f);
    if ((e = cudaMemsetAsync(counters, 0, n_counters, s)) != cudaSuccess) return e;
    p.chunk0 = a;
    p.nchunk = b - a;
    p.tiles_per_chunk = per_chunk;
    p.n_total = p.nchunk * per_chunk;
    launch_pairs(l, p, s, tza, tzb, twb, tvh, tza, tza, tzb, tzb, tmf);
    launches += 2;
    a = b;
  }
  count_launches(launches);
  return cudaGetLastError();
}

cudaError_t inplace_bwd_run(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                            const void* Vhat, const void* W_chunks, const void* dO,
                            const float* dW_final, void* dZ, void* dVhat, float* dW,
                            const bool* reset, void* ws, unsigned* err, cudaStream_t s) {
  const int NC = T / C;
  // with document resets the running adjoint lives in the workspace and dW collects it at every
  // document start; without, dW is the running adjoint itself
  float* R = reset ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) +
                                              inplace_workspace(T, d_ff, d_model, C, false))
                   : dW;
  // bf16 eta Wh_{i+1}: two rotating copies
  __nv_bfloat16* Mb = static_cast<__nv_bfloat16*>(ws);
  int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 2 * (size_t)d_model * d_ff * 2);
  CUtensorMap tza, tzb, tmb, tdx, tdo, tvk, twc, tmbn, tmf;
  if (!make_tmap_f32(&tmf, R, d_ff, d_model, d_ff, MBOX, BM) ||
      !make_tmap_bf16(&tza, Z, d_ff, T, d_ff, BK, BM) ||
      !make_tmap_bf16(&tzb, Z, d_ff, T, d_ff, 64, BK) ||
      !make_tmap_bf16(&tmb, Mb, d_ff, 2 * (size_t)d_model, d_ff, BK, BN / 2) ||
      !make_tmap_bf16(&tdx, dO, d_model, T, d_model, 64, BK) ||
      !make_tmap_bf16(&tdo, dO, d_model, T, d_model, BK, BM) ||
      !make_tmap_bf16(&tvk, Vhat, d_model, T, d_model, BK, BM) ||
      !make_tmap_bf16(&twc, W_chunks, d_ff, (size_t)NC * d_model, d_ff, 64, BK) ||
      !make_tmap_bf16(&tmbn, Mb, d_ff, 2 * (size_t)d_model, d_ff, 64, BK))
    return cudaErrorInvalidValue;
  Launch l;
  cudaError_t e = prepare(&l);
  if (e != cudaSuccess) return e;
  const size_t nW = (size_t)d_model * d_ff;
  if (reset && (e = cudaMemsetAsync(dW, 0, nW * sizeof(float), s)) != cudaSuccess) return e;
  const int n_mblk = (d_model + PTM - 1) / PTM, n_nblk = (d_ff + BN - 1) / BN;
  const size_t n_counters = ((size_t)NC + 2 * (size_t)NC * (n_mblk + n_nblk)) * sizeof(int);
  Params p{};
  p.C = C;
  p.d_ff = d_ff;
  p.d_model = d_model;
  p.n_row_n = (d_model + BN - 1) / BN;
  p.n_dz_n = (d_ff + BN - 1) / BN;
  p.n_upd_n = (d_ff + BN - 1) / BN;
  pair_tiles(p, C, C, d_model);
  p.kb_row = d_ff / BK;
  p.kb_dz_split = d_model / BK;
  p.kb_dz = 2 * p.kb_dz_split;
  p.kb_upd = C / BK;
  p.acc_scale = 1.f;
  p.copy_scale = lr;
  p.M = R;
  p.Mb = Mb;
  p.Orow = static_cast<__nv_bfloat16*>(dVhat);
  p.Odz = static_cast<__nv_bfloat16*>(dZ);
  p.err = err;
  // One persistent launch per document, the last document first, each from its last chunk;
  // each tile waits for the tiles of the chunk after it that it depends on. The last document's
  // adjoint starts from dW_final; an earlier document's from zero (the next document restarted
  // from the initial W), and each document's adjoint at its first chunk joins dW.
  p.persistent = 2;
  p.upd_col_major = 1;
  p.dz_first = 1;
  p.n_mblk = n_mblk;
  p.n_nblk = n_nblk;
  p.done = counters + NC;
  p.counter = counters;
  const int per_chunk = p.n_total;
  int launches = 0;
  for (int b = NC; b > 0;) {
    int a = b - 1;
    while (a > 0 && !(reset && reset[a])) --a;
    const int first = (b - a - 1) & 1;  // copy slot the document's last chunk reads
    if (b == NC && dW_final) {
      e = cudaMemcpyAsync(R, dW_final, nW * sizeof(float), cudaMemcpyDeviceToDevice, s);
      if (e != cudaSuccess) return e;
      to_bf16_kernel<<<l.sms * 4, 256, 0, s>>>(dW_final, Mb + first * nW, nW, lr);
      ++launches;
    } else if ((e = cudaMemsetAsync(R, 0, nW * sizeof(float), s)) != cudaSuccess ||
               (e = cudaMemsetAsync(Mb + first * nW, 0, nW * 2, s)) != cudaSuccess) {
      return e;
    }
    if ((e = cudaMemsetAsync(counters, 0, n_counters, s)) != cudaSuccess) return e;
    p.chunk0 = a;
    p.nchunk = b - a;
    p.tiles_per_chunk = per_chunk;
    p.n_total = p.nchunk * per_chunk;
    launch_pairs(l, p, s, tza, tzb, tmb, tdx, tdo, tvk, twc, tmbn, tmf);
    ++launches;
    if (reset) {
      add_kernel<<<l.sms * 4, 256, 0, s>>>(dW, R, nW / 4);
      ++launches;
    }
    b = a;
  }
  count_launches(launches);
  return cudaGetLastError();
}

size_t inplace_target_workspace(int T, int d) { return (size_t)T * d * 2 + 256; }

// Vhat = Conv1D(X0) W_target: the convolution into bf16 Y (workspace), then Y W_target as one
// launch of dz-kind tiles (A = Y K-major, B = W_target [d rows, d cols] MN-major, K = d).
cudaError_t inplace_target_run(int T, int d, int k, const void* X0, const float* conv_w,
                               const void* W_target, void* Vhat, void* ws, unsigned* err,
                               cudaStream_t s) {
  __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(ws);
  int* counter = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + (size_t)T * d * 2);
  CUtensorMap ty, twt;
  if (!make_tmap_bf16(&ty, Y, d, T, d, BK, BM) || !make_tmap_bf16(&twt, W_target, d, d, d, 64, BK))
    return cudaErrorInvalidValue;
  Launch l;
  cudaError_t e = prepare(&l);
  if (e != cudaSuccess) return e;
  if ((e = conv_fwd_launch(static_cast<const __nv_bfloat16*>(X0), conv_w, Y, T, d, k, s)))
    return e;
  e = cudaMemsetAsync(counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  Params p{};
  p.chunk = 0;
  p.C = T;  // one "chunk": the whole sequence
  p.d_ff = d;
  p.d_model = d;
  p.n_dz_n = (d + BN - 1) / BN;
  pair_tiles(p, 0, T, 0);
  p.kb_dz = d / BK;
  p.kb_dz_split = p.kb_dz;  // every k-block from the first operand pair
  p.wb_next_row0 = -1;
  p.Odz = static_cast<__nv_bfloat16*>(Vhat);
  p.counter = counter;
  p.err = err;
  launch_pairs(l, p, s, ty, ty, ty, ty, ty, ty, twt, twt, ty);
  count_launches(2);
  return cudaGetLastError();
}

// Y (bf16), dY (bf16) and the per-run tap partial sums.
size_t inplace_target_bwd_workspace(int T, int d, int k) {
  const size_t nrun = T / kRun;
  return 2 * (size_t)T * d * 2 + nrun * k * d * 4 + 256;
}

// Backward of inplace_target_run for J = <dVhat, Vhat>: recompute Y; one launch of row tiles
// dY = dVhat W_target^T (A = dVhat K-major, B = W_target [d rows, d cols] K-major over its
// columns) and update tiles dW_target = Y^T dVhat (MN-major both, K = T); then the transposed
// convolution (dX0) with the tap partials, and their reduction (dconv_w).
cudaError_t inplace_target_bwd_run(int T, int d, int k, const void* X0, const float* conv_w,
                                   const void* W_target, const void* dVhat, void* dX0,
                                   float* dconv_w, float* dW_target, void* ws, unsigned* err,
                                   cudaStream_t s) {
  const int nrun = T / kRun;
  __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* dY = Y + (size_t)T * d;
  float* part = reinterpret_cast<float*>(dY + (size_t)T * d);
  int* counter = reinterpret_cast<int*>(part + (size_t)nrun * k * d);
  CUtensorMap tdv_k, tdv_n, twt_k, ty_n, tmf;
  if (!make_tmap_f32(&tmf, dW_target, d, d, d, MBOX, BM) ||
      !make_tmap_bf16(&tdv_k, dVhat, d, T, d, BK, BM) ||
      !make_tmap_bf16(&tdv_n, dVhat, d, T, d, 64, BK) ||
      !make_tmap_bf16(&twt_k, W_target, d, d, d, BK, BN / 2) ||
      !make_tmap_bf16(&ty_n, Y, d, T, d, 64, BK))
    return cudaErrorInvalidValue;
  Launch l;
  cudaError_t e = prepare(&l);
  if (e != cudaSuccess) return e;
  if ((e = conv_fwd_launch(static_cast<const __nv_bfloat16*>(X0), conv_w, Y, T, d, k, s)))
    return e;
  if ((e = cudaMemsetAsync(dW_target, 0, (size_t)d * d * sizeof(float), s)) != cudaSuccess ||
      (e = cudaMemsetAsync(counter, 0, sizeof(int), s)) != cudaSuccess)
    return e;
  Params p{};
  p.chunk = 0;
  p.C = T;
  p.d_ff = d;
  p.d_model = d;
  p.n_row_n = (d + BN - 1) / BN;
  p.n_upd_n = (d + BN - 1) / BN;
  pair_tiles(p, T, 0, d);
  p.kb_row = d / BK;
  p.kb_upd = T / BK;
  p.wb_next_row0 = -1;
  p.acc_scale = 1.f;
  p.copy_scale = 1.f;
  p.M = dW_target;
  p.Orow = dY;
  p.counter = counter;
  p.err = err;
  launch_pairs(l, p, s, tdv_k, tdv_n, twt_k, ty_n, tdv_k, tdv_k, tdv_n, tdv_n, tmf);
  if ((e = conv_bwd_launch(static_cast<const __nv_bfloat16*>(X0), conv_w, dY,
                           static_cast<__nv_bfloat16*>(dX0), part, dconv_w, T, d, k, s)))
    return e;
  count_launches(4);
  return cudaGetLastError();
}

// dW = lr Vhat^T Z over all T tokens (the update of every chunk summed; the update is
// associative): one launch of update tiles with K = T into the zeroed float32 dW.
cudaError_t inplace_delta_run(int T, int d_ff, int d_model, float lr, const void* Z,
                              const void* Vhat, float* dW, void* ws, unsigned* err,
                              cudaStream_t s) {
  int* counter = static_cast<int*>(ws);
  CUtensorMap tzb, tvh, tmf;
  if (!make_tmap_bf16(&tzb, Z, d_ff, T, d_ff, 64, BK) ||
      !make_tmap_bf16(&tvh, Vhat, d_model, T, d_model, 64, BK) ||
      !make_tmap_f32(&tmf, dW, d_ff, d_model, d_ff, MBOX, BM))
    return cudaErrorInvalidValue;
  Launch l;
  cudaError_t e = prepare(&l);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dW, 0, (size_t)d_model * d_ff * sizeof(float), s)) != cudaSuccess ||
      (e = cudaMemsetAsync(counter, 0, sizeof(int), s)) != cudaSuccess)
    return e;
  Params p{};
  p.chunk = 0;
  p.C = T;
  p.d_ff = d_ff;
  p.d_model = d_model;
  p.n_upd_n = (d_ff + BN - 1) / BN;
  pair_tiles(p, 0, 0, d_model);
  p.kb_upd = T / BK;
  p.wb_next_row0 = -1;
  p.acc_scale = lr;
  p.copy_scale = 1.f;
  p.M = dW;
  p.counter = counter;
  p.err = err;
  launch_pairs(l, p, s, tzb, tzb, tzb, tvh, tzb, tzb, tzb, tzb, tmf);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t add_f32_run(float* dst, const float* src, size_t n, cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  add_kernel<<<sms * 4, 256, 0, s>>>(dst, src, n / 4);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tttk
