// fa_tc.cuh -- the tcgen05 dataflow: decode attention with the two skinny
// products on the 5th-generation tensor cores (bf16 K/V, head_dim 128,
// segments of 9 to 32 query rows: several query tokens per request, or GQA
// groups wider than 8).
//
// "FlashDecoding++" explainer, section "Flat GEMM optimization": with few
// query rows per kv head the products are flat (small M); padding them to a
// large tile wastes the tensor core.  Here the KV tile supplies the large
// dimension instead: tokens are M = 128 of the score product and head
// dimensions are M = 128 of the output product, while the 16 or 32 query
// rows are N.
//
//   S^T[token][row] = K[token][:] . Q[row][:]        (TMEM, fp32)
//   P = exp2(S^T * scale - m_row)                     (softmax warps, fp32)
//   O^T[dim][row]   = V^T[dim][:] . P^T[:][row]       (TMEM, fp32; P as bf16
//                                                      hi + lo parts)
//
// Warp roles of a block (one per SM):
//   warp 0  producer: bulk tensor copies of K and V tiles (128 tokens,
//           landing as [8-token group][plane][8][128 bytes], 128-byte
//           swizzle: one copy per page of a paged pool, 16 copies of 8 rows
//           of contiguous K/V) and of each piece's query rows;
//   warp 1  allocates tensor memory; one lane issues every score product
//           and commits its completion to mbarriers;
//   warps 2-9  the softmax group: two row halves of four warps, each half
//           covering the four TMEM lane quarters.  Thread (half, t) reads
//           token t's scores of its half of the rows from TMEM, keeps their
//           running max (uniform over the group, rescaled only past an 8
//           log2-unit slack), writes its part of P to shared memory, and
//           reads back dimension t of each tile's O^T for the same rows,
//           accumulating it in fp32 registers;
//   warp 10 one lane issues every output product (so that a tile's output
//           product, and the release of its V slot, never waits behind the
//           next tile's K copy).
// The scores of tile i + 1 are computed while the softmax group works on tile
// i; the output product of tile i runs while the scores of tile i + 1 are
// read.  Every wait is bounded (2 s, then the block records the wait and
// unwinds); tensor memory is freed on every exit path.
#pragma once

#include "fa_kernel.cuh"

namespace fa {

template <int NR>
struct TcCfg {
  static_assert(NR == 16 || NR == 32, "16 or 32 query rows per segment (padded)");
  static constexpr int D = 128;
  static constexpr int N = NR;
  static constexpr int T = 128;            // tokens per tile: M of the score product
  static constexpr int ROWB = 2 * D;       // bf16 row bytes
  static constexpr int NP = ROWB / 128;    // 128-byte planes per row
  static constexpr int BOX_T = 8;          // tokens per copy
  static constexpr int GROUP_BYTES = BOX_T * ROWB;  // one copy: [NP][8][128]
  static constexpr int BOXES = T / BOX_T;
  static constexpr int TILE_BYTES = T * ROWB;
  // V slots are held until the output product (after the softmax of the
  // tile), K slots only until the score product: 32 rows keep 2 K slots to
  // afford a third V slot
  static constexpr int KSTAGES = NR <= 16 ? 3 : 2;
  static constexpr int VSTAGES = 3;
  static constexpr int QSLOT_BYTES = NP * N * 128;  // [NP][N rows][128]
  static constexpr int P_BYTES = T * N * 2;         // P hi (or lo) of a tile: [T][N] bf16
  static constexpr int SG_WARPS = 8;   // softmax group: two row halves x 4 TMEM lane quarters
  static constexpr int PV_WARP = 2 + SG_WARPS;  // issues the output products
  static constexpr int THREADS = 32 * (PV_WARP + 1);
  static constexpr uint32_t TMEM_COLS = 128;        // S[2] and O[2], N columns each
  static constexpr uint32_t P_LAYOUT = N == 32 ? tc::kSwizzle64 : tc::kSwizzle32;
  // shared memory, from a 1024-aligned base
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KSTAGES * TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + VSTAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_Q + 2 * QSLOT_BYTES;
  static constexpr int OFF_BAR = OFF_P + 4 * P_BYTES;  // P[2], hi + lo each
  static constexpr int NBARS = 2 * KSTAGES + 2 * VSTAGES + 16;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
  static constexpr int OFF_RED = OFF_TMEM + 16;    // [4][N] floats
  static constexpr int OFF_ALPHA = OFF_RED + 4 * N * 4;  // [2][N] floats
  static constexpr int OFF_PAGES = OFF_ALPHA + 2 * N * 4;  // 64 page ids
  static constexpr int OFF_SCHED = OFF_PAGES + 256;
  static constexpr size_t bytes(int batch) {
    return 1024 + static_cast<size_t>(OFF_SCHED) + static_cast<size_t>(3 * batch + 1) * 4;
  }
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && P_BYTES % 1024 == 0, "operand alignment");
};

// Warp-wide reduction of N values per lane, one row per value: afterwards
// lane l holds the reduction of row l % N over the warp (N <= 32).  Each
// step halves the values a lane keeps, so the warp spends N - 1 shuffles
// plus one per remaining lane bit, instead of 5 N.
template <int N, bool MAX>
__device__ __forceinline__ float warp_rows_reduce(float (&v)[N], int lane) {
#pragma unroll
  for (int k = N / 2; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int j = 0; j < k; ++j) {
      const float send = up ? v[j] : v[j + k];
      const float keep = up ? v[j + k] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, k);
      v[j] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float r = v[0];
#pragma unroll
  for (int k = N; k < 32; k <<= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, r, k);
    r = MAX ? fmaxf(r, o) : r + o;
  }
  return r;
}

template <int NR>
__global__ void __launch_bounds__(TcCfg<NR>::THREADS, 1)
    fa_decode_tc_kernel(const __grid_constant__ KernelArgs a) {
  using C = TcCfg<NR>;
  constexpr int D = C::D, T = C::T, N = C::N, NP = C::NP;
  constexpr int KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw);
  const uint32_t kring = sbase + C::OFF_K, vring = sbase + C::OFF_V, qslots = sbase + C::OFF_Q;
  const uint32_t p_buf = sbase + C::OFF_P;  // tile j: hi at p_buf + (j % 2) * 2 P_BYTES, lo after it
  const uint32_t kfull0 = sbase + C::OFF_BAR, kempty0 = kfull0 + 8 * KS;
  const uint32_t vfull0 = kempty0 + 8 * KS, vempty0 = vfull0 + 8 * VS;
  const uint32_t qfull0 = vempty0 + 8 * VS, qempty0 = qfull0 + 16;
  const uint32_t sfull0 = qempty0 + 16, sfree0 = sfull0 + 16;
  const uint32_t pfull0 = sfree0 + 16, ofull0 = pfull0 + 16, ofree0 = ofull0 + 16;
  const uint32_t done_bar = ofree0 + 16, done_o = done_bar + 8;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + C::OFF_TMEM);
  float* s_red = reinterpret_cast<float*>(base + C::OFF_RED);
  float* s_alpha = reinterpret_cast<float*>(base + C::OFF_ALPHA);
  int* s_pages = reinterpret_cast<int*>(base + C::OFF_PAGES);
  int* s_start = reinterpret_cast<int*>(base + C::OFF_SCHED);
  const int B = a.batch, H = a.kv_heads;
  int* s_len = s_start + B;
  int* s_pre = s_len + B;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {  // kernel parameters: safe to touch before the wait below
    prefetch_tensormap(&a.kmap);
    prefetch_tensormap(&a.vmap);
    prefetch_tensormap(&a.qmap);
  }
  // nothing in global memory is touched before the preceding work is done
  asm volatile("griddepcontrol.wait;" ::: "memory");

  load_lengths(a, s_start, s_len);
  if (warp == 1) {  // the whole warp allocates; the address lands in s_tmem
    tc::tmem_alloc(smem_addr(s_tmem), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(kfull0 + 8 * s, 1);
      mbar_init(kempty0 + 8 * s, 1);   // the commit of the tile's score product
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(vfull0 + 8 * s, 1);
      mbar_init(vempty0 + 8 * s, 1);   // the commit of the tile's output product
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(qfull0 + 8 * s, 1);
      mbar_init(qempty0 + 8 * s, 1);   // the commit of the piece's last score product
      mbar_init(sfull0 + 8 * s, 1);
      mbar_init(sfree0 + 8 * s, C::SG_WARPS);  // one arrival per softmax warp
      mbar_init(ofull0 + 8 * s, 1);
      mbar_init(ofree0 + 8 * s, C::SG_WARPS);
      mbar_init(pfull0 + 8 * s, C::SG_WARPS);
    }
    mbar_init(done_bar, 1);
    mbar_init(done_o, 1);
    fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *s_tmem;
  if (warp == 0) tile_prefix(a, s_len, s_pre, T, lane);
  __syncthreads();

  const int P = gridDim.x, c = blockIdx.x;
  const PieceIter it = block_run(a, s_pre, P, c);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 32) write_boundary_record(a, it, s_pre, s_len, T, c);

  const int GK = a.group, Q = a.q_len;
  const int G = GK * Q;  // rows of a segment (<= N)

  if (warp == 0) {
    // ================= producer
    const uint64_t pol = l2_evict_first_policy();
    const int ps = a.paged ? (1 << a.page_shift) : 0;
    const int win_paged = !a.paged ? 1 : (ps >= T ? 63 * (ps / T) : (64 * ps) / T);
    int ks = 0, vs = 0;
    uint32_t kph = 0, vph = 0;
    int kissued = 0, vissued = 0, pq = 0;  // tiles whose K / V copies went out
    bool ok = true;
    auto load_ids = [&](const Piece& p, int w, int (&v)[2], bool (&in)[2]) {
      const int np = (s_len[p.b] + ps - 1) >> a.page_shift;
      const int pb = (w * T) >> a.page_shift;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e = pb + half * 32 + lane;
        in[half] = e < np;
        v[half] = in[half] ? __ldg(a.page_table + static_cast<long long>(p.b) * a.pt_stride + e) : -1;
      }
    };
    auto store_ids = [&](const int (&v)[2], const bool (&in)[2]) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        int x = v[half];
        if (in[half] && (x < 0 || static_cast<long long>(x) >= a.kv_rows)) {
          atomicOr(a.status, kFlagBadPage);
          x = -1;  // its copies read out of range: zeros, no memory access
        }
        s_pages[half * 32 + lane] = in[half] ? x : -1;
      }
    };
    PieceIter itp = it;
    Piece pc;
    bool have = next_piece(itp, pc, s_pre, s_len, B, H, a.window_u, T);
    int w0 = have ? pc.t0 : 0;
    if (have && a.paged) {
      int v[2];
      bool in[2];
      load_ids(pc, w0, v, in);
      store_ids(v, in);
      __syncwarp();
    }
    while (ok && have) {
      const int L = s_len[pc.b];
      if (w0 == pc.t0 && lane == 0) {
        // the piece's query rows, plane by plane and token by token, into
        // q slot pq % 2 as [plane][row][128 bytes] (128-byte swizzle)
        const int qs = pq & 1;
        const uint32_t qpar = ((pq >> 1) & 1) ^ 1u;
        if (!mbar_wait(qempty0 + 8 * qs, qpar, kWaitLimitNs)) {
          record_timeout(a.status, 5, pq, qs, qpar, qempty0 + 8 * qs);
          ok = false;
        } else {
          mbar_arrive_expect_tx(qfull0 + 8 * qs, static_cast<uint32_t>(G * C::ROWB));
          for (int i = 0; i < Q; ++i) {
            const int row = (pc.b * Q + i) * a.qo_heads + pc.h * GK;
#pragma unroll
            for (int p = 0; p < NP; ++p)
              tma_load_3d(qslots + qs * C::QSLOT_BYTES + p * (N * 128) + i * GK * 128, &a.qmap,
                          qfull0 + 8 * qs, 0, row, p, pol);
          }
        }
      }
      if (w0 == pc.t0) {
        ++pq;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      const int w1 = a.paged && w0 + win_paged < pc.t1 ? w0 + win_paged : pc.t1;
      PieceIter itn = itp;
      Piece pn = pc;
      int nw0 = w1;
      bool nhave = true;
      if (w1 >= pc.t1) {
        nhave = next_piece(itn, pn, s_pre, s_len, B, H, a.window_u, T);
        nw0 = nhave ? pn.t0 : 0;
      }
      int nv[2] = {-1, -1};
      bool nin[2] = {false, false};
      if (a.paged && nhave) load_ids(pn, nw0, nv, nin);  // in flight during the issue loop
      const int npages = a.paged ? (L + ps - 1) >> a.page_shift : 0;
      const int pbase = a.paged ? (w0 * T) >> a.page_shift : 0;
      {
        // Copies of a tile: contiguous rows, 16 copies of 8 rows (row
        // s_start + token); paged, one copy per page of up to 128 tokens,
        // addressed by 8-row group of the pool (a page holds page_size
        // consecutive rows; a missing page reads zeros from a negative
        // group).  Lane j of the warp issues copy j, so one instruction sends
        // all of a tile's copies; lane 0 waits for the slot and arms its
        // barrier first.
        const int cp = a.paged ? (ps < T ? ps : T) : C::BOX_T;  // tokens per copy
        const int ncp = T / cp;
        for (int tt = w0; tt < w1 && ok; ++tt) {
          int crd = 0;  // this lane's copy: contiguous, first row; paged, first 8-row group
          if (lane < ncp) {
            const int tok = tt * T + lane * cp;
            if (!a.paged) {
              crd = s_start[pc.b] + tok;
            } else {
              const int pidx = tok >> a.page_shift;
              const int page = (pidx < npages && pidx - pbase < 64) ? s_pages[pidx - pbase] : -1;
              crd = (page * ps + (tok & (ps - 1))) >> 3;
            }
          }
          const uint32_t dst_off = static_cast<uint32_t>(lane * (cp / 8) * C::GROUP_BYTES);
          if (lane == 0) {
            if (!mbar_wait(kempty0 + 8 * ks, kph ^ 1u, kWaitLimitNs)) {
              record_timeout(a.status, 1, kissued, ks, kph ^ 1u, kempty0 + 8 * ks);
              ok = false;
            } else {
              mbar_arrive_expect_tx(kfull0 + 8 * ks, C::TILE_BYTES);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (lane < ncp) {
            const uint32_t dst = kring + ks * C::TILE_BYTES + dst_off;
            if (a.paged)
              tma_load_5d(dst, &a.kmap, kfull0 + 8 * ks, 0, 0, 0, pc.h, crd, pol);
            else
              tma_load_4d(dst, &a.kmap, kfull0 + 8 * ks, 0, crd, 0, pc.h, pol);
          }
          ++kissued;
          if (lane == 0) {
            if (!mbar_wait(vempty0 + 8 * vs, vph ^ 1u, kWaitLimitNs)) {
              record_timeout(a.status, 8, vissued, vs, vph ^ 1u, vempty0 + 8 * vs);
              ok = false;
            } else {
              mbar_arrive_expect_tx(vfull0 + 8 * vs, C::TILE_BYTES);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (lane < ncp) {
            const uint32_t dst = vring + vs * C::TILE_BYTES + dst_off;
            if (a.paged)
              tma_load_5d(dst, &a.vmap, vfull0 + 8 * vs, 0, 0, 0, pc.h, crd, pol);
            else
              tma_load_4d(dst, &a.vmap, vfull0 + 8 * vs, 0, crd, 0, pc.h, pol);
          }
          ++vissued;
          if (++ks == KS) {
            ks = 0;
            kph ^= 1u;
          }
          if (++vs == VS) {
            vs = 0;
            vph ^= 1u;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      __syncwarp();
      if (a.paged && nhave) store_ids(nv, nin);
      __syncwarp();
      if (w1 >= pc.t1) {
        have = nhave;
        pc = pn;
        itp = itn;
        w0 = nw0;
      } else {
        w0 = w1;
      }
    }
    // drain: every issued copy has landed before the block may exit
    if (lane == 0) {
      for (int j = kissued - KS < 0 ? 0 : kissued - KS; j < kissued; ++j) {
        const int st = j % KS;
        const uint32_t par = (j / KS) & 1;
        if (!mbar_wait(kfull0 + 8 * st, par, kWaitLimitNs)) {
          record_timeout(a.status, 2, j, st, par, kfull0 + 8 * st);
          break;
        }
      }
      for (int j = vissued - VS < 0 ? 0 : vissued - VS; j < vissued; ++j) {
        const int st = j % VS;
        const uint32_t par = (j / VS) & 1;
        if (!mbar_wait(vfull0 + 8 * st, par, kWaitLimitNs)) {
          record_timeout(a.status, 9, j, st, par, vfull0 + 8 * st);
          break;
        }
      }
      for (int k = pq - 2 < 0 ? 0 : pq - 2; k < pq; ++k) {
        if (!mbar_wait(qfull0 + 8 * (k & 1), (k >> 1) & 1, kWaitLimitNs)) {
          record_timeout(a.status, 7, k, k & 1, (k >> 1) & 1, qfull0 + 8 * (k & 1));
          break;
        }
      }
    }
    return;
  }

  constexpr uint32_t kIdescS = tc::idesc_bf16(128, N, false, false);
  constexpr uint32_t kIdescO = tc::idesc_bf16(128, N, true, true);
  const uint32_t tS = tmem, tO = tmem + 2 * N;  // column offsets of S[2] and O[2]

  if (warp == 1 || warp == C::PV_WARP) {
    // ================= tcgen05.mma issue: lane 0 of warp 1 the score
    // products, lane 0 of PV_WARP the output products, so that a tile's
    // output product (and the release of its V slot) never waits behind the
    // next tile's K copy
    if (lane == 0 && warp == C::PV_WARP) {
      bool ok = true;
      PieceIter itv = it;
      Piece pc;
      int j = 0;
      while (ok && next_piece(itv, pc, s_pre, s_len, B, H, a.window_u, T)) {
        const int n = pc.t1 - pc.t0;
        for (int t = 0; t < n && ok; ++t, ++j) {
          // output product of tile j: O^T[j % 2] = V_j^T . (P_hi + P_lo)^T
          const int vsl = j % VS;
          if (!mbar_wait(vfull0 + 8 * vsl, (j / VS) & 1, kWaitLimitNs)) {
            record_timeout(a.status, 11, j, vsl, (j / VS) & 1, vfull0 + 8 * vsl);
            ok = false;
            break;
          }
          if (!mbar_wait(pfull0 + 8 * (j & 1), (j >> 1) & 1, kWaitLimitNs)) {
            record_timeout(a.status, 12, j, j & 1, (j >> 1) & 1, pfull0 + 8 * (j & 1));
            ok = false;
            break;
          }
          if (j >= 2 && !mbar_wait(ofree0 + 8 * (j & 1), ((j - 2) >> 1) & 1, kWaitLimitNs)) {
            record_timeout(a.status, 13, j, j & 1, ((j - 2) >> 1) & 1, ofree0 + 8 * (j & 1));
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d = tO + (j & 1) * N;
          // V^T: dims as M (64-dim atoms one plane = 1024 bytes apart),
          // tokens as K (8-token groups GROUP_BYTES apart); P^T: rows as N
          // (2N bytes a token), tokens as K (8-token groups 16 N apart).
          // Descriptors of step k: the first one plus the step's offset / 16.
          const uint32_t a_lo = tc::smem_desc_lo(vring + vsl * C::TILE_BYTES, 1024);
          const uint32_t b_lo = tc::smem_desc_lo(p_buf + (j & 1) * 2 * C::P_BYTES, T * 2 * N);
          constexpr uint32_t a_hi = tc::smem_desc_hi(C::GROUP_BYTES, tc::kSwizzle128);
          constexpr uint32_t b_hi = tc::smem_desc_hi(8 * 2 * N, C::P_LAYOUT);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int k = 0; k < T / 16; ++k) {
              const uint64_t ad = tc::desc_of(a_lo + k * (2 * C::GROUP_BYTES / 16), a_hi);
              const uint64_t bd = tc::desc_of(b_lo + part * (C::P_BYTES / 16) + k * (16 * 2 * N / 16), b_hi);
              tc::mma_bf16_ss(d, ad, bd, kIdescO, part > 0 || k > 0);
            }
          }
          tc::commit(ofull0 + 8 * (j & 1));
          tc::commit(vempty0 + 8 * vsl);
        }
      }
      // every product issued has completed before tensor memory is freed
      tc::commit(done_o);
      if (!mbar_wait(done_o, 0, kWaitLimitNs)) record_timeout(a.status, 17, j, 1, 0, done_o);
    }
    if (lane == 0 && warp == 1) {
      bool ok = true;
      int i = 0, pcount = 0;
      PieceIter itm = it;
      Piece pc;
      while (ok && next_piece(itm, pc, s_pre, s_len, B, H, a.window_u, T)) {
        const int qs = pcount & 1;
        if (!mbar_wait(qfull0 + 8 * qs, (pcount >> 1) & 1, kWaitLimitNs)) {
          record_timeout(a.status, 14, pcount, qs, (pcount >> 1) & 1, qfull0 + 8 * qs);
          ok = false;
          break;
        }
        const int n = pc.t1 - pc.t0;
        for (int t = 0; t < n && ok; ++t, ++i) {
          const int ksl = i % KS;
          if (!mbar_wait(kfull0 + 8 * ksl, (i / KS) & 1, kWaitLimitNs)) {
            record_timeout(a.status, 15, i, ksl, (i / KS) & 1, kfull0 + 8 * ksl);
            ok = false;
            break;
          }
          if (i >= 2 && !mbar_wait(sfree0 + 8 * (i & 1), ((i - 2) >> 1) & 1, kWaitLimitNs)) {
            record_timeout(a.status, 16, i, i & 1, ((i - 2) >> 1) & 1, sfree0 + 8 * (i & 1));
            ok = false;
            break;
          }
          tc::fence_after_sync();
          // scores S^T[i % 2] = K_i . Q^T: tokens as M (8-token groups
          // GROUP_BYTES apart), query rows as N (8-row groups 1024 bytes
          // apart); a k-step of 16 dims is 32 bytes into a 128-byte plane
          const uint32_t a_lo = tc::smem_desc_lo(kring + ksl * C::TILE_BYTES, 16);
          const uint32_t b_lo = tc::smem_desc_lo(qslots + qs * C::QSLOT_BYTES, 16);
          constexpr uint32_t a_hi = tc::smem_desc_hi(C::GROUP_BYTES, tc::kSwizzle128);
          constexpr uint32_t b_hi = tc::smem_desc_hi(1024, tc::kSwizzle128);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * (N * 128) + (kk & 3) * 32;
            const uint64_t ad = tc::desc_of(a_lo + off / 16, a_hi);
            const uint64_t bd = tc::desc_of(b_lo + qoff / 16, b_hi);
            tc::mma_bf16_ss(tS + (i & 1) * N, ad, bd, kIdescS, kk > 0);
          }
          tc::commit(sfull0 + 8 * (i & 1));
          tc::commit(kempty0 + 8 * ksl);
          if (t == n - 1) tc::commit(qempty0 + 8 * qs);
        }
        ++pcount;
      }
      // every product issued has completed before tensor memory is freed
      tc::commit(done_bar);
      if (!mbar_wait(done_bar, 0, kWaitLimitNs)) record_timeout(a.status, 17, i, 0, 0, done_bar);
    }
    named_barrier_sync(2, 64 + 32 * C::SG_WARPS);
    if (warp == 1) {
      tc::fence_after_sync();
      tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
    return;
  }

  // ================= softmax group (warps 2..9)
  // Two row halves of 4 warps each: the warps of a half cover the four TMEM
  // lane quarters (a warp reads the lanes of quarter warp % 4), so thread
  // (half, tok) handles token tok of a tile for rows [r0, r0 + NH), and
  // dimension tok of the output for the same rows.
  constexpr int NH = N / 2;
  constexpr int SGT = 32 * C::SG_WARPS;       // softmax-group threads
  const int quarter = warp & 3;              // this warp's quarter of TMEM lanes
  const int tok = quarter * 32 + lane;       // token of a tile; dim of an output row
  const int half = (warp - 2) >> 2;          // 0 or 1
  const int r0 = half * NH;                  // first row of this half
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  float* red = s_red + half * 4 * NH;        // this half's [quarter][NH] scratch
  write_empty_results(a, it, s_len, G, D, c, P, tid - 64, SGT);
  // parameters in registers for the tile loop
  const float sscale = a.score_scale, cap = a.cap_l2;
  const int W = a.window, WU = a.window_u;
  // a finite start for the running max: exp2(x - m) is then 0 for a masked
  // score (x = -inf) without a select, and the first finite score of a row
  // always passes the slack test (which rescales by exp2(-1e30 - x) = 0)
  constexpr float kMStart = -1e30f;

  float acc[NH], l[NH], m[NH];
  bool alive = true;     // this warp's waits have all succeeded
  int i = 0;             // tile of the block's sequence
  int pending = -1;      // tile whose output product is not yet accumulated
  uint32_t resc = 0;     // bit j % 2: tile j rescaled the running max (alpha in s_alpha[j % 2])
  PieceIter its = it;
  Piece pc;

  // Accumulates O^T of tile j (this thread's dimension, its rows).  A
  // failed wait only stops this warp's work: the group agrees to stop at its
  // next barrier (bar_any on !alive), so every named barrier below is
  // reached by all the group's threads or by none.
  auto take_o = [&](int j) {
    if (!alive) return;
    const bool ok = mbar_wait(ofull0 + 8 * (j & 1), (j >> 1) & 1, kWaitLimitNs);
    if (!ok && lane == 0) record_timeout(a.status, 18, j, j & 1, (j >> 1) & 1, ofull0 + 8 * (j & 1));
    if (!__all_sync(0xffffffffu, ok)) {  // tcgen05.ld is warp-collective
      alive = false;
      return;
    }
    float o[NH];
    tc::ld_32x32b<NH>(tO + lanes + (j & 1) * N + r0, o);
    tc::wait_ld();
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(ofree0 + 8 * (j & 1));
    if (resc & (1u << (j & 1))) {
      const float* al = s_alpha + (j & 1) * N + r0;
#pragma unroll
      for (int r = 0; r < NH; ++r) acc[r] = fmaf(acc[r], al[r], o[r]);
    } else {
#pragma unroll
      for (int r = 0; r < NH; ++r) acc[r] += o[r];
    }
  };
  // A bounded wait of the whole warp: false (and the wait recorded) if any
  // lane gave up.
  auto warp_wait = [&](uint32_t bar, uint32_t parity, uint32_t site, int idx, int stage) {
    const bool ok = mbar_wait(bar, parity, kWaitLimitNs);
    if (!ok && lane == 0) record_timeout(a.status, site, idx, stage, parity, bar);
    return __all_sync(0xffffffffu, ok);
  };

  bool stop = false;
  bool have = next_piece(its, pc, s_pre, s_len, B, H, a.window_u, T);
  while (!stop && have) {
    const int L = s_len[pc.b];
    const int lo = (WU > 0 && L > WU) ? L - WU : 0;  // keys some row sees: [lo, L)
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      acc[r] = 0.f;
      l[r] = 0.f;
      m[r] = kMStart;
    }
    const int n = pc.t1 - pc.t0;
    for (int t = 0; t < n; ++t, ++i) {
      __syncwarp();
      if (bar_any(1, SGT, !alive)) {  // the group stops together
        stop = true;
        break;
      }
      const int pos0 = (pc.t0 + t) * T;
      const int pos = pos0 + tok;
      float x[NH];
      if (warp_wait(sfull0 + 8 * (i & 1), (i >> 1) & 1, 19, i, i & 1)) {
        tc::ld_32x32b<NH>(tS + lanes + (i & 1) * N + r0, x);
        tc::wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(sfree0 + 8 * (i & 1));
      } else {
        alive = false;
#pragma unroll
        for (int r = 0; r < NH; ++r) x[r] = 0.f;
      }
      // The rows that see this thread's key: query token q (rows q GK ..
      // q GK + GK - 1) sees keys below L - Q + 1 + q and, with a window, from
      // L - Q + 1 + q - W on, so the rows form one range [rlo, rlo + rspan).
      const int base = pos - L + Q;
      const int qlo = base > 0 ? base : 0;
      const int qhi = W > 0 ? (base + W < Q ? base + W : Q) : Q;
      const int rlo = qlo * GK - r0;  // relative to this half's first row
      const uint32_t rspan = qhi > qlo ? static_cast<uint32_t>((qhi - qlo) * GK) : 0u;
      // scale (log2 units), soft-cap, then the masks
#pragma unroll
      for (int r = 0; r < NH; ++r) x[r] *= sscale;
      if (cap > 0.f) {
#pragma unroll
        for (int r = 0; r < NH; ++r) x[r] = cap * tanhf(x[r] / cap);
      }
      bool need = false;
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        x[r] = static_cast<uint32_t>(r - rlo) < rspan ? x[r] : -CUDART_INF_F;
        need |= x[r] - m[r] > kRescaleSlack;
      }
      __syncwarp();
      const bool slow = bar_any(1, SGT, need);
      resc &= ~(1u << (i & 1));
      if (slow) {
        // the tile's maximum of each of this half's rows over the 128 tokens
        float v[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) v[r] = x[r];
        const float wmax = warp_rows_reduce<NH, true>(v, lane);
        if (lane < NH) red[quarter * NH + lane] = wmax;
        named_barrier_sync(1, SGT);
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          const float tm = fmaxf(fmaxf(red[r], red[NH + r]), fmaxf(red[2 * NH + r], red[3 * NH + r]));
          float al = 1.f;
          if (tm - m[r] > kRescaleSlack) {
            al = exp2_approx(m[r] - tm);  // from the start value: 0
            m[r] = tm;
          }
          l[r] *= al;
          if (tok == r) s_alpha[(i & 1) * N + r0 + r] = al;
        }
        resc |= 1u << (i & 1);
        named_barrier_sync(1, SGT);  // s_alpha written; the scratch read by all
      }
      // P = exp2(x - m) (0 for a masked key), its row sums, and the bf16
      // hi / lo parts
      uint32_t ph[NH / 2], pl[NH / 2];
#pragma unroll
      for (int r = 0; r < NH; r += 2) {
        const float p0 = exp2_approx(x[r] - m[r]);
        const float p1 = exp2_approx(x[r + 1] - m[r + 1]);
        l[r] += p0;
        l[r + 1] += p1;
        const uint32_t h = pack_bf16x2(p0, p1);
        ph[r / 2] = h;
        pl[r / 2] = pack_bf16x2(p0 - bf16lo(h), p1 - bf16hi(h));
      }
      if (!alive) continue;
      // V rows of keys outside [lo, L) may hold anything (NaN included) and
      // meet P = 0 in the product: zeroed once the tile has landed (by the
      // first half; every half's P arrival precedes the product)
      if (half == 0 && (pos0 < lo || pos0 + T > L)) {
        const bool out = pos < lo || pos >= L;
        if (__any_sync(0xffffffffu, out)) {
          const int vsl = i % VS;
          if (!warp_wait(vfull0 + 8 * vsl, (i / VS) & 1, 20, i, vsl)) {
            alive = false;
            continue;
          }
          if (out) {
            const uint32_t row = vring + vsl * C::TILE_BYTES + (tok >> 3) * C::GROUP_BYTES + (tok & 7) * 128;
#pragma unroll
            for (int p = 0; p < NP; ++p)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch) sts128(row + p * 1024 + ch * 16, make_uint4(0, 0, 0, 0));
          }
        }
      }
      // P^T of tile i into buffer i % 2 (free: the output product of tile
      // i - 2 was waited for when its O was read), N rows of a token
      // contiguous (2N bytes), 16-byte chunks of 8 rows swizzled by the
      // address bits above them (64- or 32-byte swizzle); this half writes
      // its chunks
      {
        constexpr int CH = NH / 8;  // 16-byte chunks of this half's rows
        const int sel = N == 32 ? ((tok >> 1) & 3) : ((tok >> 2) & 1);
        const uint32_t hi_buf = p_buf + (i & 1) * 2 * C::P_BYTES;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
          const uint32_t off = tok * (2 * N) + (((half * CH + ch) ^ sel) * 16);
          sts128(hi_buf + off, make_uint4(ph[4 * ch], ph[4 * ch + 1], ph[4 * ch + 2], ph[4 * ch + 3]));
          sts128(hi_buf + C::P_BYTES + off,
                 make_uint4(pl[4 * ch], pl[4 * ch + 1], pl[4 * ch + 2], pl[4 * ch + 3]));
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull0 + 8 * (i & 1));
      if (pending >= 0) take_o(pending);
      pending = i;
    }
    if (stop) break;
    // ---- piece end: the next piece's schedule (looked up while the last
    // tile's output product runs), the last tile's output, the row sums,
    // the results
    Piece pn;
    const bool have_next = next_piece(its, pn, s_pre, s_len, B, H, a.window_u, T);
    if (pending >= 0) take_o(pending);
    pending = -1;
    __syncwarp();
    if (bar_any(1, SGT, !alive)) break;  // also: every reader of the scratch is done
    float lsum[NH];
    {
      float v[NH];
#pragma unroll
      for (int r = 0; r < NH; ++r) v[r] = l[r];
      const float wsum = warp_rows_reduce<NH, false>(v, lane);
      if (lane < NH) red[quarter * NH + lane] = wsum;
      named_barrier_sync(1, SGT);
#pragma unroll
      for (int r = 0; r < NH; ++r) lsum[r] = (red[r] + red[NH + r]) + (red[2 * NH + r] + red[3 * NH + r]);
    }
    const bool whole = pc.n_pieces == 1;
    const int slot_idx = c + pc.seg;
    // O = acc / l and the row's lse (natural log).  Straight-line code with
    // one pointer stepped row by row: this runs once per piece, so its
    // instructions are cold, and each cache line of them fetched while the
    // copies saturate memory stalls the whole group.
    float val[NH];
    float my_l = 0.f, my_m = 0.f;  // row r0 + tok's sum and max (tok < NH): its lse
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      val[r] = lsum[r] > 0.f ? acc[r] * rcp_approx(lsum[r]) : 0.f;
      my_l = tok == r ? lsum[r] : my_l;
      my_m = tok == r ? m[r] : my_m;
    }
    const float my_lse = my_l > 0.f ? (my_m + __log2f(my_l)) * kLn2 : -CUDART_INF_F;
    const int nrows = G - r0 < NH ? G - r0 : NH;  // rows of this half that exist
    if (whole) {
      // segment row rr is query token rr / GK, head rr % GK of the group
      int hd = r0 % GK;
      const size_t row0 = (static_cast<size_t>(pc.b) * Q + r0 / GK) * a.qo_heads +
                          static_cast<size_t>(pc.h) * GK + hd;
      size_t po = row0 * D + tok;  // element of out for row r0 + r
      const size_t jump = static_cast<size_t>(a.qo_heads - GK) * D;  // last head of a token -> first of the next
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        if (r < nrows) a.out[po] = bf16_bits(val[r]);
        po += D;
        if (++hd == GK) {
          hd = 0;
          po += jump;
        }
      }
      if (tok < nrows && a.lse != nullptr) {
        const int rr = r0 + tok;
        a.lse[(static_cast<size_t>(pc.b) * Q + rr / GK) * a.qo_heads +
              static_cast<size_t>(pc.h) * GK + rr % GK] = my_lse;
      }
    } else if (FA_CHECK(a.status, slot_idx < a.max_partials, 402, slot_idx)) {
      float* po = a.part_o + (static_cast<size_t>(slot_idx) * G + r0) * D + tok;
#pragma unroll
      for (int r = 0; r < NH; ++r)
        if (r < nrows) po[r * D] = val[r];
      if (tok < nrows) a.part_lse[static_cast<size_t>(slot_idx) * G + r0 + tok] = my_lse;
    }
    pc = pn;
    have = have_next;
  }
  tc::fence_before_sync();
  named_barrier_sync(2, 64 + SGT);
}

}  // namespace fa
