// Per-warp tensor-core math of the bf16 decode kernels: one 16-token sub-tile of one KV
// head against the G query heads of its group.
//
// S = Q . K^T with m16n8k16 bf16 MMAs (query heads as the 16 rows, padded), an fp32
// online softmax in base 2, and O += P . V with P fed back from registers as the A
// operand, split into bf16 hi + lo parts so that P keeps ~16 significant bits (with at
// most 8 query rows, the lo part rides in the otherwise empty rows 8-15 of the same
// MMA).  K and V
// come from a shared-memory tile written by TMA with 128-byte swizzle: row r's 16-byte
// column chunk c sits at r*128 + ((c ^ (r & 7)) << 4) inside each 64-column chunk.
#pragma once

#include "pa_device.cuh"

namespace pa {

// TT: tokens per pipeline stage when blocks are smaller (a stage holds whole blocks).
// SPLIT: a block larger than TT is staged as TT-token parts (a stage holds part of one
// block) instead of the stage growing to the block.
template <int D_, int BS_, bool ROWS16_, int TT_ = 16, bool SPLIT_ = false>
struct TileCfg {
  static constexpr int D = D_;
  static constexpr int BS = BS_;
  static constexpr bool ROWS16 = ROWS16_;
  static constexpr int TILE_T = (SPLIT_ || BS <= TT_) ? TT_ : BS;  // tokens per pipeline stage
  static constexpr int BPS = TILE_T >= BS ? TILE_T / BS : 1;      // blocks per stage
  static constexpr int BOXR = BS < TILE_T ? BS : TILE_T;          // rows per TMA box
  static constexpr int SUBT = TILE_T / 16;           // 16-token sub-tiles per stage
  static constexpr int DCH = D / 64;                 // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = TILE_T * 128;
  static constexpr int TILE_BYTES = DCH * CHUNK_BYTES;  // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int ROWS = ROWS16 ? 16 : 8;          // query-head rows kept
  static constexpr int KSTEPS = D / 16;
  static constexpr int NT = D / 8;                      // output n-tiles of 8 columns
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 8 || BS == 16 || BS == 32, "block size");
  static_assert(TILE_T % 16 == 0 && BPS <= 4 && (TILE_T % BS == 0 || BS % TILE_T == 0),
                "stage tokens");
};

__device__ __forceinline__ uint32_t sw128(int row, int c16) {
  return static_cast<uint32_t>(row * 128 + ((c16 ^ (row & 7)) << 4));
}

// Online-softmax state and output accumulator of one warp for one (sequence, KV head).
// Lane (g = lane/4, tig = lane%4) owns rows g (and g+8 with ROWS16) and output columns
// 8j + 2tig, 8j + 2tig + 1 of every n-tile j.
//
// Q (the A operand of S = Q.K^T) is kept either in registers (QSMEM = false) or in a
// per-warp shared-memory tile of ROWS x D bf16 read by ldmatrix at every k-step
// (QSMEM = true), which frees 16-32 registers per thread.  The shared tile stores row
// r's 16-byte chunk c at r*(2D) + ((c ^ (r & 7)) << 4), so ldmatrix reads of 8 rows at
// one chunk hit 8 different bank groups.
template <class C, bool QSMEM = false>
struct WarpAcc {
  static constexpr int QROW_BYTES = C::D * 2;
  static constexpr int Q_BYTES = C::ROWS * QROW_BYTES;  // shared Q tile per warp
  float o_lo[C::NT][2];
  float o_hi[C::NT][2];
  float m_lo, m_hi, l_lo, l_hi;
  // 8-row mode (tile_t): running max and this lane's partial sum of heads 2tig, 2tig+1;
  // reduce_l() turns them into m_lo / l_lo of row g.
  float mh[2], lh[2];
  uint32_t qa[QSMEM ? 1 : C::KSTEPS][2];  // Q rows g as A fragments (register mode)
  uint32_t qh[QSMEM ? 1 : C::KSTEPS][2];  // Q rows g+8
  uint32_t qs = 0;                         // shared address of the Q tile (shared mode)

  __device__ __forceinline__ static uint32_t q_off(int r, int c16) {
    return static_cast<uint32_t>(r * QROW_BYTES + ((c16 ^ (r & 7)) << 4));
  }

  // Shared mode: copy the group's Q rows (G heads, [G][D] bf16) into the warp's tile at
  // shared address `tile` (generic pointer `tile_ptr`); rows >= G are zero.
  __device__ __forceinline__ void stage_q(const __nv_bfloat16* qrow, int G, uint8_t* tile_ptr,
                                          int lane) {
    constexpr int CPR = QROW_BYTES / 16;  // 16-byte chunks per row
    __syncwarp();  // the previous unit's ldmatrix reads of this tile are done
    for (int i = lane; i < C::ROWS * CPR; i += 32) {
      const int r = i / CPR, c = i - r * CPR;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < G) v = __ldg(reinterpret_cast<const uint4*>(qrow + r * C::D) + c);
      *reinterpret_cast<uint4*>(tile_ptr + q_off(r, c)) = v;
    }
    qs = smem_addr(tile_ptr);
    __syncwarp();
  }

  // Shared mode, asynchronous: start copying the group's Q rows into the tile at
  // `tile_ptr` with cp.async (rows >= G zero-filled), so that the load overlaps other
  // work; use_q() then waits for the copies and makes that tile the A operand.  The
  // warp must be done reading the tile (it was last used two units ago, and a
  // __syncwarp has passed since).
  __device__ __forceinline__ void prefetch_q(const __nv_bfloat16* qrow, int G,
                                             uint8_t* tile_ptr, int lane) {
    constexpr int CPR = QROW_BYTES / 16;
    for (int i = lane; i < C::ROWS * CPR; i += 32) {
      const int r = i / CPR, c = i - r * CPR;
      const bool live = r < G;
      cp_async_16_zfill(smem_addr(tile_ptr + q_off(r, c)),
                        reinterpret_cast<const uint4*>(qrow + (live ? r : 0) * C::D) + c,
                        live ? 16 : 0);
    }
    cp_async_commit();
  }

  __device__ __forceinline__ void use_q(uint8_t* tile_ptr) {
    cp_async_wait_all();
    __syncwarp();
    qs = smem_addr(tile_ptr);
  }

  // A fragments of k-step k: registers, or ldmatrix from the shared tile.
  __device__ __forceinline__ void q_frag(int k, int lane, uint32_t& a0, uint32_t& a1,
                                         uint32_t& a2, uint32_t& a3) const {
    if constexpr (QSMEM) {
      const int mi = lane >> 3, mr = lane & 7;
      if constexpr (C::ROWS16) {
        // matrices: (rows 0-7, chunk 2k), (rows 8-15, 2k), (rows 0-7, 2k+1), (rows 8-15, 2k+1)
        ldmatrix_x4(qs + q_off((mi & 1) * 8 + mr, 2 * k + (mi >> 1)), a0, a1, a2, a3);
      } else {
        // lanes 0-7: rows 0-7 at chunk 2k; lanes 8-15: rows 0-7 at chunk 2k+1
        ldmatrix_x2(qs + q_off(mr, 2 * k + (mi & 1)), a0, a2);
        a1 = 0u;
        a3 = 0u;
      }
    } else {
      a0 = qa[k][0];
      a1 = qh[k][0];
      a2 = qa[k][1];
      a3 = qh[k][1];
    }
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < C::NT; ++j) {
      o_lo[j][0] = o_lo[j][1] = 0.f;
      o_hi[j][0] = o_hi[j][1] = 0.f;
    }
    m_lo = m_hi = -INFINITY;
    mh[0] = mh[1] = -INFINITY;
    lh[0] = lh[1] = 0.f;
    l_lo = l_hi = 0.f;
  }

  // Q rows of one group (G heads, row-major [G][D] bf16); rows >= G are zero.
  __device__ __forceinline__ void load_q(const __nv_bfloat16* qrow, int G, int lane) {
    const int g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int k = 0; k < C::KSTEPS; ++k) {
      const bool lo_ok = g < G;
      qa[k][0] = lo_ok ? __ldg(reinterpret_cast<const unsigned int*>(qrow + g * C::D + 16 * k + 2 * tig)) : 0u;
      qa[k][1] = lo_ok ? __ldg(reinterpret_cast<const unsigned int*>(qrow + g * C::D + 16 * k + 8 + 2 * tig)) : 0u;
      if constexpr (C::ROWS16) {
        const bool hi_ok = g + 8 < G;
        qh[k][0] = hi_ok ? __ldg(reinterpret_cast<const unsigned int*>(qrow + (g + 8) * C::D + 16 * k + 2 * tig)) : 0u;
        qh[k][1] = hi_ok ? __ldg(reinterpret_cast<const unsigned int*>(qrow + (g + 8) * C::D + 16 * k + 8 + 2 * tig)) : 0u;
      } else {
        qh[k][0] = 0u;
        qh[k][1] = 0u;
      }
    }
  }

  // One online-softmax row update for scores x0..x3 (tokens 2tig, 2tig+1, 8+2tig, 9+2tig).
  // A masked row takes no part in this tile: its state is kept and its P is zero.
  __device__ __forceinline__ static float row_update(float x0, float x1, float x2, float x3,
                                                     float& m, float& l, uint32_t& hi0,
                                                     uint32_t& lo0, uint32_t& hi2,
                                                     uint32_t& lo2, bool masked = false) {
    constexpr unsigned kFull = 0xffffffffu;
    float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    if (masked) {
      hi0 = lo0 = hi2 = lo2 = 0u;
      return 1.f;
    }
    const float m_new = fmaxf(m, mx);
    const float alpha = exp2f(m - m_new);
    m = m_new;
    const float e0 = exp2f(x0 - m_new), e1 = exp2f(x1 - m_new);
    const float e2 = exp2f(x2 - m_new), e3 = exp2f(x3 - m_new);
    split_bf16x2(e0, e1, hi0, lo0);
    split_bf16x2(e2, e3, hi2, lo2);
    l = l * alpha + ((e0 + e1) + (e2 + e3));
    return alpha;
  }

  // Consume one staged tile (K at kbase, V at kbase + TILE_BYTES, shared addresses) with
  // `valid` tokens (1..TILE_T) inside the sequence; rows >= valid are masked (their V rows
  // must already be zero).  With ROWMASK only query rows [row_lo, row_hi) take part.
  template <bool ROWMASK = false>
  __device__ __forceinline__ void tile(uint32_t kbase, int valid, float sl2, int lane,
                                       int row_lo = 0, int row_hi = 16) {
    static_assert(!ROWMASK || C::ROWS16, "row masks are kept for 16-row tiles only");
    if constexpr (!C::ROWS16) {
      tile_t(kbase, valid, sl2, lane);
      return;
    }
    const uint32_t vbase = kbase + C::TILE_BYTES;
    const int tig = lane & 3;
    const int mi = lane >> 3, mr = lane & 7;
#pragma unroll
    for (int st = 0; st < C::SUBT; ++st) {
      const int r0 = st * 16;
      if (r0 >= valid) break;
      float s0[4] = {0.f, 0.f, 0.f, 0.f};
      float s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < C::KSTEPS; ++k) {
        const int row = r0 + (mi >> 1) * 8 + mr;
        const int d = 16 * k + (mi & 1) * 8;
        uint32_t b00, b01, b10, b11;
        ldmatrix_x4(kbase + (d >> 6) * C::CHUNK_BYTES + sw128(row, (d & 63) >> 3), b00, b01, b10,
                    b11);
        uint32_t a0, a1, a2, a3;
        q_frag(k, lane, a0, a1, a2, a3);
        mma_bf16_16816(s0[0], s0[1], s0[2], s0[3], a0, a1, a2, a3, b00, b01, s0[0], s0[1], s0[2],
                       s0[3]);
        mma_bf16_16816(s1[0], s1[1], s1[2], s1[3], a0, a1, a2, a3, b10, b11, s1[0], s1[1], s1[2],
                       s1[3]);
      }
      const int lim = valid - r0;
      const bool v0 = 2 * tig < lim, v1 = 2 * tig + 1 < lim;
      const bool v2 = 8 + 2 * tig < lim, v3 = 9 + 2 * tig < lim;
      uint32_t pa0, pa1 = 0u, pa2, pa3 = 0u;   // P hi parts (A fragment registers)
      uint32_t pr0, pr1 = 0u, pr2, pr3 = 0u;   // P lo parts
      const int gr = lane >> 2;
      const bool mask_lo = ROWMASK && (gr < row_lo || gr >= row_hi);
      const bool mask_hi = ROWMASK && (gr + 8 < row_lo || gr + 8 >= row_hi);
      const float alpha_lo =
          row_update(v0 ? s0[0] * sl2 : -INFINITY, v1 ? s0[1] * sl2 : -INFINITY,
                     v2 ? s1[0] * sl2 : -INFINITY, v3 ? s1[1] * sl2 : -INFINITY, m_lo, l_lo,
                     pa0, pr0, pa2, pr2, mask_lo);
      float alpha_hi = 1.f;
      if constexpr (C::ROWS16)
        alpha_hi = row_update(v0 ? s0[2] * sl2 : -INFINITY, v1 ? s0[3] * sl2 : -INFINITY,
                              v2 ? s1[2] * sl2 : -INFINITY, v3 ? s1[3] * sl2 : -INFINITY, m_hi,
                              l_hi, pa1, pr1, pa3, pr3, mask_hi);
#pragma unroll
      for (int j = 0; j < C::NT; ++j) {
        o_lo[j][0] *= alpha_lo;
        o_lo[j][1] *= alpha_lo;
        // with 8 rows, o_hi holds the lo-part products of the same rows (see below)
        o_hi[j][0] *= C::ROWS16 ? alpha_hi : alpha_lo;
        o_hi[j][1] *= C::ROWS16 ? alpha_hi : alpha_lo;
      }
#pragma unroll
      for (int jp = 0; jp < C::NT / 2; ++jp) {
        const int row = r0 + (mi & 1) * 8 + mr;
        const int d = 16 * jp + (mi >> 1) * 8;
        uint32_t w0, w1, w2, w3;
        ldmatrix_x4_trans(vbase + (d >> 6) * C::CHUNK_BYTES + sw128(row, (d & 63) >> 3), w0, w1,
                          w2, w3);
        if constexpr (C::ROWS16) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t a0 = half ? pr0 : pa0, a1 = half ? pr1 : pa1;
            const uint32_t a2 = half ? pr2 : pa2, a3 = half ? pr3 : pa3;
            mma_bf16_16816(o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0], o_hi[2 * jp][1], a0,
                           a1, a2, a3, w0, w1, o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0],
                           o_hi[2 * jp][1]);
            mma_bf16_16816(o_lo[2 * jp + 1][0], o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0],
                           o_hi[2 * jp + 1][1], a0, a1, a2, a3, w2, w3, o_lo[2 * jp + 1][0],
                           o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0], o_hi[2 * jp + 1][1]);
          }
        } else {
          // 8 query rows: A rows 0-7 carry P's hi part and rows 8-15 (otherwise unused)
          // its lo part, so one MMA accumulates hi.V into o_lo and lo.V into o_hi;
          // reduce_l() adds the two.
          mma_bf16_16816(o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0], o_hi[2 * jp][1], pa0,
                         pr0, pa2, pr2, w0, w1, o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0],
                         o_hi[2 * jp][1]);
          mma_bf16_16816(o_lo[2 * jp + 1][0], o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0],
                         o_hi[2 * jp + 1][1], pa0, pr0, pa2, pr2, w2, w3, o_lo[2 * jp + 1][0],
                         o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0], o_hi[2 * jp + 1][1]);
        }
      }
    }
  }

  // 8 query rows: S is computed transposed, S^T = K.Q^T, with the sub-tile's 16 tokens as
  // the MMA rows and the (up to 8) heads as its 8 columns: one MMA per k-step instead of
  // two whose rows 8-15 would be empty.  Lane (g, tig) then holds tokens g and g+8 of
  // heads 2tig and 2tig+1, so the softmax state is kept per head (mh, lh: max over the
  // 8 lanes of a column by shuffles, sums per lane until reduce_l), and movmatrix
  // transposes P back into A-operand layout (heads as rows) for O += P.V.  P.V then runs
  // as in tile(), with the lo part of P in the A rows 8-15 and its products in o_hi.
  __device__ __forceinline__ void tile_t(uint32_t kbase, int valid, float sl2, int lane) {
    constexpr unsigned kFull = 0xffffffffu;
    const uint32_t vbase = kbase + C::TILE_BYTES;
    const int g = lane >> 2;
    const int mi = lane >> 3, mr = lane & 7;
#pragma unroll
    for (int st = 0; st < C::SUBT; ++st) {
      const int r0 = st * 16;
      if (r0 >= valid) break;
      float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
      for (int k = 0; k < C::KSTEPS; ++k) {
        // A = K rows r0..r0+15 x columns 16k..16k+15; matrices (rows 0-7, 8-15) x
        // (columns 0-7, 8-15) in A-fragment order
        const int row = r0 + (mi & 1) * 8 + mr;
        const int d = 16 * k + (mi >> 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kbase + (d >> 6) * C::CHUNK_BYTES + sw128(row, (d & 63) >> 3), a0, a1, a2,
                    a3);
        // B = Q^T: Q[g][16k+2tig..] and Q[g][16k+8+2tig..] are its two fragments
        uint32_t q0, q1, q2, q3;
        q_frag(k, lane, q0, q1, q2, q3);
        mma_bf16_16816(c0, c1, c2, c3, a0, a1, a2, a3, q0, q2, c0, c1, c2, c3);
      }
      const bool va = r0 + g < valid, vb = r0 + g + 8 < valid;
      const float x0 = va ? c0 * sl2 : -INFINITY;  // token g,   head 2tig
      const float x1 = va ? c1 * sl2 : -INFINITY;  // token g,   head 2tig+1
      const float x2 = vb ? c2 * sl2 : -INFINITY;  // token g+8, head 2tig
      const float x3 = vb ? c3 * sl2 : -INFINITY;  // token g+8, head 2tig+1
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(mh[0], mx0), mn1 = fmaxf(mh[1], mx1);  // token r0 is valid
      const float al0 = exp2f(mh[0] - mn0), al1 = exp2f(mh[1] - mn1);
      mh[0] = mn0;
      mh[1] = mn1;
      const float e0 = exp2f(x0 - mn0), e1 = exp2f(x1 - mn1);
      const float e2 = exp2f(x2 - mn0), e3 = exp2f(x3 - mn1);
      lh[0] = lh[0] * al0 + (e0 + e2);
      lh[1] = lh[1] * al1 + (e1 + e3);
      uint32_t h01, l01, h23, l23;
      split_bf16x2(e0, e1, h01, l01);  // P^T row g (token), columns 2tig, 2tig+1 (heads)
      split_bf16x2(e2, e3, h23, l23);  // P^T row g+8
      // P row g (head): tokens 2tig, 2tig+1 and 8+2tig, 9+2tig, hi and lo parts
      const uint32_t pa0 = movmatrix_trans(h01), pa2 = movmatrix_trans(h23);
      const uint32_t pr0 = movmatrix_trans(l01), pr2 = movmatrix_trans(l23);
      // rescale of output row g (head g): its factor sits in the lanes with tig = g/2
      const float s0 = __shfl_sync(kFull, al0, g >> 1), s1 = __shfl_sync(kFull, al1, g >> 1);
      const float alpha = (g & 1) ? s1 : s0;
#pragma unroll
      for (int j = 0; j < C::NT; ++j) {
        o_lo[j][0] *= alpha;
        o_lo[j][1] *= alpha;
        o_hi[j][0] *= alpha;
        o_hi[j][1] *= alpha;
      }
#pragma unroll
      for (int jp = 0; jp < C::NT / 2; ++jp) {
        const int row = r0 + (mi & 1) * 8 + mr;
        const int d = 16 * jp + (mi >> 1) * 8;
        uint32_t w0, w1, w2, w3;
        ldmatrix_x4_trans(vbase + (d >> 6) * C::CHUNK_BYTES + sw128(row, (d & 63) >> 3), w0, w1,
                          w2, w3);
        mma_bf16_16816(o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0], o_hi[2 * jp][1], pa0,
                       pr0, pa2, pr2, w0, w1, o_lo[2 * jp][0], o_lo[2 * jp][1], o_hi[2 * jp][0],
                       o_hi[2 * jp][1]);
        mma_bf16_16816(o_lo[2 * jp + 1][0], o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0],
                       o_hi[2 * jp + 1][1], pa0, pr0, pa2, pr2, w2, w3, o_lo[2 * jp + 1][0],
                       o_lo[2 * jp + 1][1], o_hi[2 * jp + 1][0], o_hi[2 * jp + 1][1]);
      }
    }
  }

  // Finish the unit's sums: the per-lane partial row sums over the 4 lanes of each row;
  // with 8 rows (tile_t), the per-head state over the 8 lanes of each column, moved to
  // row g's m_lo / l_lo, and the lo-part products (o_hi) added into o_lo.  Call once,
  // before reading the outputs.
  __device__ __forceinline__ void reduce_l() {
    constexpr unsigned kFull = 0xffffffffu;
    if constexpr (!C::ROWS16) {
#pragma unroll
      for (int j = 0; j < C::NT; ++j) {
        o_lo[j][0] += o_hi[j][0];
        o_lo[j][1] += o_hi[j][1];
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lh[0] += __shfl_xor_sync(kFull, lh[0], off);
        lh[1] += __shfl_xor_sync(kFull, lh[1], off);
      }
      const int g = (threadIdx.x & 31) >> 2;
      const float m0 = __shfl_sync(kFull, mh[0], g >> 1), m1 = __shfl_sync(kFull, mh[1], g >> 1);
      const float s0 = __shfl_sync(kFull, lh[0], g >> 1), s1 = __shfl_sync(kFull, lh[1], g >> 1);
      m_lo = (g & 1) ? m1 : m0;
      l_lo = (g & 1) ? s1 : s0;
      return;
    }
    l_lo += __shfl_xor_sync(kFull, l_lo, 1);
    l_lo += __shfl_xor_sync(kFull, l_lo, 2);
    if constexpr (C::ROWS16) {
      l_hi += __shfl_xor_sync(kFull, l_hi, 1);
      l_hi += __shfl_xor_sync(kFull, l_hi, 2);
    }
  }
};

// Zero the V rows [valid, TILE_T) of a staged tile (their slots may hold anything), then
// order those generic-proxy writes before later TMA writes to the same stage.
template <class C>
__device__ __forceinline__ void zero_tail_rows(uint8_t* stage_ptr, int valid, int lane) {
  uint8_t* vt = stage_ptr + C::TILE_BYTES;
  const int nchunks = (C::TILE_T - valid) * C::DCH * 8;
  for (int i = lane; i < nchunks; i += 32) {
    const int r = valid + i / (C::DCH * 8);
    const int rem = i % (C::DCH * 8);
    *reinterpret_cast<uint4*>(vt + (rem >> 3) * C::CHUNK_BYTES + r * 128 + (rem & 7) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  __syncwarp();
}

}  // namespace pa
