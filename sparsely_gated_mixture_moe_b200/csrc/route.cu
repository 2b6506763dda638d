// Router product fused with the gate.
//
// Scores (Shazeer et al., "Noisy Top-K Gating"; Switch Transformer, switch_routing):
//   softmax gating: l = x.W_g (+ bias); choose the k largest l;
//                   renorm: G = Softmax(KeepTopK(l, k)); else gate = softmax(l)[chosen]
//   noisy gating:   H = l + n * Softplus(x.W_noise); choose the k largest H;
//                   G = Softmax(KeepTopK(H, k))
// Ties go to the lowest expert index (the running top list ranks equal scores by
// expert index, so lists built over disjoint expert sets merge exactly).  For noisy
// gating (or when Importance is asked for) the kernel also forms, per token tile, the
// partial sums of Importance = sum_t G(x_t) and
// Load_i = sum_t Phi((l_i - kth_excluding(H, k, i)) / Softplus((x.W_noise)_i))
// ("Load-Balancing-Losses"); a second kernel adds the partials in a fixed order, so
// results are bit-reproducible (no floating-point atomics).
//
// bf16 (route_tc_kernel): persistent over token tiles, warp-specialised.  Warp 0 streams
// x tiles [128 x 64] and W_g (and W_noise) tiles [E_pad x 64] with TMA into a ring of
// shared-memory stages; one thread of warp 1 issues tcgen05.mma (M=128, N=E_pad) into
// one of two TMEM accumulator buffers (one when noisy gating's two products fill TMEM);
// 4*G gate warps (G = 4, or 2 when k > 4) take a finished buffer, run gate_tile and hand
// it back, so one tile's gate overlaps the next tile's loads.  Tiles are 128 tokens, or
// 64 tokens loaded into both halves of the MMA operand when 128-token tiles would fill
// at most half of the SMs.  In gate_tile each thread owns one token row of its warp's
// TMEM lane quarter and 16-column slices of experts interleaved across the column
// groups, read with one tcgen05.ld + wait per slice; it keeps a running top-(k+1) list
// (branch-free insertion) and the running softmax in registers, then one column group
// merges the partial lists through shared memory and writes the outputs.  The logits
// never touch HBM.
// fp32 (gate_f32_kernel): the logits come from the SIMT product into the workspace and
// the same gate code reads them back (one token per thread, G = 1).
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kRouteBM = 128;

// Tiles of the router: 128 tokens, or 64 ("half tiles") when 128-token tiles would leave
// most SMs idle.  The partial Importance/Load sums are kept per tile, so the workspace
// is sized for 64-token tiles.
int route_blocks(int64_t T) { return static_cast<int>((T + 63) / 64); }

struct GateArgs {
  int64_t T;
  int E, k, noisy, renorm;
  int groups, k_primary;  // hierarchical gating (groups > 0): E experts in groups of E/groups
  const float* noise;
  const float* bias;
  int32_t* topk_idx;
  float* topk_gate;
  uint8_t* near_tie;
  float* partials;  // [gridDim.x][2][E] or null
  // Scores kept for later kernels, all [E, T] (expert-major, so a warp's 32 tokens store
  // 128 contiguous bytes), or null: each token's clean logits (bias added) in lw and, for
  // noisy gating, Softplus(x.W_noise) in sw, the noisy scores H in hw and the k-th and
  // (k+1)-th H [2, T] in kw.  Written for noisy gating with Importance/Load asked for on
  // the tensor-core path (split = 1: the gate leaves the sums to importance_load_kernel,
  // which forms them over the whole grid) and for the training forward (the backward
  // reads them instead of recomputing the router).
  float* lw;
  float* sw;
  float* hw;
  float* kw;
  int split;
};

// Softplus(z) = max(z, 0) + log(1 + e^-|z|), with the fast exponential and logarithm:
// for u = e^-|z| < 1/64 log(1 + u) is its Taylor polynomial to u^4 (truncation below
// 1/64^5 / 5 relative), else __logf(1 + u), whose absolute error on [1, 2] is below
// 2^-21.  The result is within about 5e-7 of the exact value, far inside the margin at
// which the top-k choice counts as a near tie (1e-4).
__device__ __forceinline__ float softplus_f(float z) {
  const float u = __expf(-fabsf(z));
  const float l1p = (u < 0.015625f)
                        ? u * (1.0f - u * (0.5f - u * (0.33333333f - u * 0.25f)))
                        : __logf(1.0f + u);
  return fmaxf(z, 0.0f) + l1p;
}

// Descending list of the KM+1 largest (score, expert) pairs seen; a pair ranks higher
// when its score is larger, or equal with a lower expert index.  Insertion order does
// not matter, so partial lists over disjoint expert sets merge exactly.
template <int KM>
struct TopList {
  float v[KM + 1];
  int i[KM + 1];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int s = 0; s <= KM; ++s) {
      v[s] = -INFINITY;
      i[s] = 0x7fffffff;
    }
  }
  // Branch-free insertion of a score that arrives after every equal score already in the
  // list (ascending expert order): it displaces the entries it strictly exceeds.  Every
  // slot is computed from the old list, so the KM+1 updates are independent.
  __device__ __forceinline__ void push(float cv, int ci) {
#pragma unroll
    for (int q = KM; q >= 1; --q) {
      const bool up = cv > v[q - 1];
      const bool here = cv > v[q];
      const float nv = up ? v[q - 1] : (here ? cv : v[q]);
      const int ni = up ? i[q - 1] : (here ? ci : i[q]);
      v[q] = nv;
      i[q] = ni;
    }
    const bool first = cv > v[0];
    v[0] = first ? cv : v[0];
    i[0] = first ? ci : i[0];
  }
};

// Merges the list (ov, oi), over experts disjoint from t's, into t: afterwards t holds
// the KM+1 highest-ranked pairs of both.  A pair's place in the union is its place in
// its own list plus the number of pairs of the other list ranked above it; the
// (KM+1)^2 comparisons are independent of one another, unlike insertion one pair at a
// time.  Empty slots (-inf, 0x7fffffff) rank below every expert's score and never above
// one another, so they only fill the places the experts leave.
template <int KM>
__device__ __forceinline__ void merge_top(TopList<KM>& t, const float (&ov)[KM + 1],
                                          const int (&oi)[KM + 1]) {
  int ra[KM + 1], rb[KM + 1];
#pragma unroll
  for (int p = 0; p <= KM; ++p) {
    ra[p] = p;
    rb[p] = p;
  }
#pragma unroll
  for (int p = 0; p <= KM; ++p)
#pragma unroll
    for (int q = 0; q <= KM; ++q) {
      const bool above = ov[q] > t.v[p] || (ov[q] == t.v[p] && oi[q] < t.i[p]);
      ra[p] += above ? 1 : 0;
      rb[q] += above ? 0 : 1;
    }
  float nv[KM + 1];
  int ni[KM + 1];
#pragma unroll
  for (int r = 0; r <= KM; ++r) {
    nv[r] = -INFINITY;
    ni[r] = 0x7fffffff;
#pragma unroll
    for (int p = 0; p <= KM; ++p) {
      nv[r] = (ra[p] == r) ? t.v[p] : nv[r];
      ni[r] = (ra[p] == r) ? t.i[p] : ni[r];
    }
#pragma unroll
    for (int q = 0; q <= KM; ++q) {
      nv[r] = (rb[q] == r) ? ov[q] : nv[r];
      ni[r] = (rb[q] == r) ? oi[q] : ni[r];
    }
  }
#pragma unroll
  for (int r = 0; r <= KM; ++r) {
    t.v[r] = nv[r];
    t.i[r] = ni[r];
  }
}

// Shared-memory bytes gate_tile needs for 128*G gate threads.
__host__ __device__ constexpr int gate_smem_bytes(int KM, int G, int E) {
  return G * 128 * (KM + 1) * 8     // partial lists (scores, experts)
         + G * 128 * 8              // partial softmax (max, sum)
         + 128 * (2 * KM + 2) * 4   // final experts, gates, k-th and (k+1)-th score
         + 4 * 2 * E * 4            // per-lane-quarter column sums (Importance, Load)
         + E * 4                    // logit bias (zeros when there is none)
         + 64;
}

// Bias of each expert's logit into shared memory (zeros without a bias), by `nthreads`
// threads of which this is number `tid`; the caller synchronises before gate_tile.
__device__ __forceinline__ void load_bias_smem(const GateArgs& g, uint8_t* smem, int KM, int G,
                                               int tid, int nthreads) {
  float* sbias = reinterpret_cast<float*>(smem + gate_smem_bytes(KM, G, g.E) - 64 - g.E * 4);
  for (int e = tid; e < g.E; e += nthreads) sbias[e] = g.bias ? __ldg(g.bias + e) : 0.0f;
}

// Sum of v[j] over the 32 lanes of a warp for each of the 8 columns j, as a
// reduce-scatter: each step halves the columns a lane keeps and adds its partner's
// half; afterwards lane l holds the sum of column 4*(l&1) + 2*((l>>1)&1) + ((l>>2)&1)
// (lanes 0..7 hold all eight).  The order of additions is fixed, so the sums are
// reproducible.
__device__ __forceinline__ float warp_colsum8(const float (&v)[8], int lane) {
  const bool b0 = lane & 1, b1 = lane & 2, b2 = lane & 4;
  float w4[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float send = b0 ? v[j] : v[j + 4];
    const float keep = b0 ? v[j + 4] : v[j];
    w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  float w2[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = b1 ? w4[j] : w4[j + 2];
    const float keep = b1 ? w4[j + 2] : w4[j];
    w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  float w1 = (b2 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? w2[0] : w2[1], 4);
  w1 += __shfl_xor_sync(0xffffffffu, w1, 8);
  w1 += __shfl_xor_sync(0xffffffffu, w1, 16);
  return w1;
}
__device__ __forceinline__ int colsum8_column(int lane) {
  return 4 * (lane & 1) + 2 * ((lane >> 1) & 1) + ((lane >> 2) & 1);
}

// The gate for one tile of 128 tokens (tokens 128*tile ...), computed by 128*G gate
// threads: the thread in lane l of gate warp w owns token row r = 32*q + l, where q is
// the TMEM lane quarter its warp may read, and the expert columns c = W*grp + W*G*i + j
// (0 <= j < W) of its column group grp = w / 4 (the four warps of a group cover the
// four quarters).
// `fetch(c, l, z)` fills l[0..W-1] with the raw clean logits x.W_g of experts c..c+W-1
// of this thread's token (c a multiple of W) and z[0..W-1] with x.W_noise (noisy
// gating); it is called by all 32 lanes of a warp together and waits once for its
// loads.  `sync()` is a barrier over the 128*G gate threads.  Each W-column slice is
// scored from registers: its maximum updates the running softmax (one rescale per
// slice), and a group of 8 scores enters the top list by branch-free insertion unless
// no lane of the warp has one above its current (k+1)-th score.  The column groups'
// partial lists then merge pairwise in log2(column groups) rounds (merge_top).  The
// logit bias has been loaded into shared memory (load_bias_smem) by the caller.
template <int KM, int G, int W, class Fetch, class Sync>
__device__ __forceinline__ void gate_tile(const Fetch& fetch, const Sync& sync, int q, int grp,
                                          int gtid, int64_t tile, bool half, const GateArgs& g,
                                          uint8_t* smem) {
  const int lane = gtid & 31;
  // half tiles: 64 tokens whose rows fill both halves of the MMA operand, so quarters q
  // and q+2 hold the same tokens and split their experts (2G column groups)
  const int ntok = half ? 64 : 128;
  const int row = half ? (q & 1) * 32 + lane : q * 32 + lane;
  const int CG = half ? 2 * G : G;
  const int cgrp = half ? grp * 2 + (q >> 1) : grp;
  const int64_t t0 = tile * ntok;
  const int64_t t = t0 + row;
  const bool valid = t < g.T;
  const int E = g.E, k = g.k;
  const float* noise_row = (g.noisy && valid) ? g.noise + t * E : nullptr;
  // 8 noise draws per step, as two 16-byte loads when the rows keep 16-byte alignment
  const bool noise_vec = g.noisy && (E % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.noise) & 15u) == 0);
  auto load_noise8 = [&](int c, float (&nz)[8]) {
    if (noise_row != nullptr && noise_vec && c + 8 <= E) {
      const float4 u0 = __ldg(reinterpret_cast<const float4*>(noise_row + c));
      const float4 u1 = __ldg(reinterpret_cast<const float4*>(noise_row + c + 4));
      nz[0] = u0.x; nz[1] = u0.y; nz[2] = u0.z; nz[3] = u0.w;
      nz[4] = u1.x; nz[5] = u1.y; nz[6] = u1.z; nz[7] = u1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) nz[j] = (noise_row != nullptr && c + j < E) ? __ldg(noise_row + c + j) : 0.0f;
    }
  };
  const bool noisy = g.noisy != 0;
  const bool full_softmax = !noisy && !g.renorm;

  float* pv = reinterpret_cast<float*>(smem);                    // [G][128][KM+1]
  int* pi = reinterpret_cast<int*>(pv + G * 128 * (KM + 1));     // [G][128][KM+1]
  float* pm = reinterpret_cast<float*>(pi + G * 128 * (KM + 1)); // [G][128]
  float* ps = pm + G * 128;                                      // [G][128]
  int* fid = reinterpret_cast<int*>(ps + G * 128);               // [128][KM]
  float* fgate = reinterpret_cast<float*>(fid + 128 * KM);       // [128][KM]
  float* fkth = fgate + 128 * KM;                                // [128][2]
  float* qsum = fkth + 128 * 2;                                  // [4][2][E]

  const float* sbias = qsum + 4 * 2 * E;                       // [E]

  // ---- pass 1: partial top-(k+1), maximum and softmax sum over this thread's experts
  auto scores = [&](int cs, float (&sc)[W]) {
    float l[W], z[W];
    fetch(cs, l, z);
#pragma unroll
    for (int g8 = 0; g8 < W / 8; ++g8) {
      float nz[8];
      if (noisy) load_noise8(cs + 8 * g8, nz);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int jj = 8 * g8 + j, e = cs + jj;
        float sv = -INFINITY;
        if (e < E) {
          sv = l[jj] + sbias[e];
          if (noisy) {
            const float sp = softplus_f(z[jj]);
            const float li = sv;
            sv = __fmaf_rn(nz[j], sp, sv);  // H
            if (g.lw != nullptr && valid) {
              g.lw[e * g.T + t] = li;
              g.sw[e * g.T + t] = sp;
              g.hw[e * g.T + t] = sv;
            }
          } else if (g.lw != nullptr && valid) {
            g.lw[e * g.T + t] = sv;
          }
        }
        sc[jj] = sv;
      }
    }
  };
  TopList<KM> top;
  top.init();
  float thr = -INFINITY;  // the current (k+1)-th score: values below it cannot enter the list
  float m = -INFINITY, ssum = 0.0f;
#pragma unroll 1
  for (int cs = cgrp * W; cs < E; cs += W * CG) {
    {
      float sc[W];
      scores(cs, sc);
      float gm8[W / 8];
#pragma unroll
      for (int g8 = 0; g8 < W / 8; ++g8) {
        const float* v8 = sc + 8 * g8;
        gm8[g8] = fmaxf(fmaxf(fmaxf(v8[0], v8[1]), fmaxf(v8[2], v8[3])),
                        fmaxf(fmaxf(v8[4], v8[5]), fmaxf(v8[6], v8[7])));
      }
      float sm = gm8[0];
#pragma unroll
      for (int g8 = 1; g8 < W / 8; ++g8) sm = fmaxf(sm, gm8[g8]);
      if (full_softmax) {
        const float nm = fmaxf(m, sm);
        float add = 0.0f;
#pragma unroll
        for (int jj = 0; jj < W; ++jj) add += (cs + jj < E) ? __expf(sc[jj] - nm) : 0.0f;
        ssum = ssum * __expf(m - nm) + add;  // exp(-inf) = 0 before the first slice
        m = nm;
      } else {
        m = fmaxf(m, sm);
      }
#pragma unroll
      for (int g8 = 0; g8 < W / 8; ++g8) {
        // skipped by the whole warp when no lane has a score above its (k+1)-th
        if (__any_sync(0xffffffffu, gm8[g8] > thr)) {
#pragma unroll
          for (int j = 0; j < 8; ++j) top.push(sc[8 * g8 + j], cs + 8 * g8 + j);
          // the list is sorted, so the maximum over slots >= k is slot k
          thr = -INFINITY;
#pragma unroll
          for (int q2 = 0; q2 <= KM; ++q2)
            if (q2 >= k) thr = fmaxf(thr, top.v[q2]);
        }
      }
    }
  }
#pragma unroll
  for (int s2 = 0; s2 <= KM; ++s2) {
    pv[(cgrp * ntok + row) * (KM + 1) + s2] = top.v[s2];
    pi[(cgrp * ntok + row) * (KM + 1) + s2] = top.i[s2];
  }
  pm[cgrp * ntok + row] = m;
  ps[cgrp * ntok + row] = ssum;
  sync();

  // ---- merge the CG partial results of each token pairwise (column group c takes in
  // c + s for s = CG/2, CG/4, ..., 1), then group 0 writes the outputs
#pragma unroll 1
  for (int s = CG >> 1; s >= 1; s >>= 1) {
    if (cgrp < s) {
      const int o = (cgrp + s) * ntok + row;
      float ov[KM + 1];
      int oi[KM + 1];
#pragma unroll
      for (int s2 = 0; s2 <= KM; ++s2) {
        ov[s2] = pv[o * (KM + 1) + s2];
        oi[s2] = pi[o * (KM + 1) + s2];
      }
      merge_top<KM>(top, ov, oi);
      if (full_softmax) {
        const float m2 = pm[o], s2v = ps[o];
        if (m2 != -INFINITY) {
          const float nm = fmaxf(m, m2);
          ssum = (m == -INFINITY ? 0.0f : ssum * expf(m - nm)) + s2v * expf(m2 - nm);
          m = nm;
        }
      }
      if (s > 1) {
        const int own = cgrp * ntok + row;
#pragma unroll
        for (int s2 = 0; s2 <= KM; ++s2) {
          pv[own * (KM + 1) + s2] = top.v[s2];
          pi[own * (KM + 1) + s2] = top.i[s2];
        }
        pm[own] = m;
        ps[own] = ssum;
      }
    }
    if (s > 1) sync();
  }
  if (cgrp == 0) {
    float gate[KM];
    if (full_softmax) {
#pragma unroll
      for (int j = 0; j < KM; ++j) gate[j] = (j < k) ? expf(top.v[j] - m) / ssum : 0.0f;
    } else {
      float den = 0.0f;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        gate[j] = (j < k) ? expf(top.v[j] - top.v[0]) : 0.0f;
        den += gate[j];
      }
#pragma unroll
      for (int j = 0; j < KM; ++j) gate[j] /= den;
    }
    // k-th and (k+1)-th largest scores.  The list is sorted, so they are the minimum of
    // the first k entries and the maximum of the rest; written as predicated min/max (a
    // select on j == k would become an indexed load and push the list to local memory).
    float kth = INFINITY, kth1 = -INFINITY;
#pragma unroll
    for (int j = 0; j <= KM; ++j) {
      if (j < k) kth = fminf(kth, top.v[j]);
      else kth1 = fmaxf(kth1, top.v[j]);
    }
    if (valid) {
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k) {
          g.topk_idx[t * k + j] = top.i[j];
          g.topk_gate[t * k + j] = gate[j];
        }
      if (g.near_tie) g.near_tie[t] = (k < E && (kth - kth1) <= 1e-4f) ? 1 : 0;
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      fid[row * KM + j] = (j < k) ? top.i[j] : -1;
      fgate[row * KM + j] = gate[j];
    }
    fkth[row * 2 + 0] = kth;
    fkth[row * 2 + 1] = kth1;
    if (g.kw != nullptr && valid) {
      g.kw[t] = kth;
      g.kw[g.T + t] = kth1;
    }
  }
  if (g.partials == nullptr || g.split) {  // uniform across the gate threads
    sync();                                        // the lists are reused by the next tile
    return;
  }
  sync();

  // ---- pass 2: Importance and Load partial sums over this tile's tokens
  const float kth = fkth[row * 2 + 0], kth1 = fkth[row * 2 + 1];
  int myid[KM];  // this token's chosen experts (-1 past k) and their gates
  float myg[KM];
#pragma unroll
  for (int jj = 0; jj < KM; ++jj) {
    myid[jj] = fid[row * KM + jj];
    myg[jj] = fgate[row * KM + jj];
  }
#pragma unroll 1
  for (int cs = cgrp * W; cs < E; cs += W * CG) {
    {
      float gi[W], pl[W];
#pragma unroll
      for (int jj = 0; jj < W; ++jj) {
        gi[jj] = 0.0f;
        pl[jj] = 0.0f;
      }
      {
        float l[W], z[W];
        fetch(cs, l, z);
#pragma unroll
        for (int g8 = 0; g8 < W / 8; ++g8) {
          float nz[8];
          if (noisy) load_noise8(cs + 8 * g8, nz);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int jj = 8 * g8 + j, e = cs + jj;
            if (valid && e < E) {
              if (noisy && k < E) {
                // recomputed exactly as in pass 1, so H >= kth means "among the top k"
                const float li = l[jj] + sbias[e];
                const float sp = softplus_f(z[jj]);
                const float H = __fmaf_rn(nz[j], sp, li);
                const float ex = (H >= kth) ? kth1 : kth;  // kth_excluding(H, k, e)
                // Phi((l_e - kth_excluding) / Softplus(z_e))
                pl[jj] = 0.5f + 0.5f * erf_as7126(__fdividef(li - ex, sp) * 0.70710678118654752f);
              }
#pragma unroll
              for (int q3 = 0; q3 < KM; ++q3)
                if (myid[q3] == e) gi[jj] = myg[q3];
            }
          }
        }
      }
      // column sums over the warp's 32 tokens, 8 columns at a time
#pragma unroll
      for (int g8 = 0; g8 < W / 8; ++g8) {
        float a8[8], b8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          a8[j] = gi[8 * g8 + j];
          b8[j] = pl[8 * g8 + j];
        }
        const float si = warp_colsum8(a8, lane);
        const float sl = warp_colsum8(b8, lane);
        const int col = cs + 8 * g8 + colsum8_column(lane);
        if (lane < 8 && col < E) {
          qsum[(q * 2 + 0) * E + col] = si;
          qsum[(q * 2 + 1) * E + col] = sl;
        }
      }
    }
  }
  sync();
  for (int e = gtid; e < E; e += 128 * G) {
    float si = 0.0f, sl = 0.0f;
    // half tiles: column e was summed by the quarter pair of its column group only
    const int q0 = half ? 2 * (((e / W) % CG) & 1) : 0, q1 = half ? q0 + 2 : 4;
    for (int qq = q0; qq < q1; ++qq) {
      si += qsum[(qq * 2 + 0) * E + e];
      sl += qsum[(qq * 2 + 1) * E + e];
    }
    g.partials[(tile * 2 + 0) * E + e] = si;
    g.partials[(tile * 2 + 1) * E + e] = sl;
  }
  sync();  // qsum and the lists are reused by the next tile
}

// The hierarchical gate for one tile of 128 tokens, by 128 threads (one token row each;
// the thread in lane l of the warp reading TMEM lane quarter q owns row 32*q + l).  The
// score columns are the primary gate's over the A = g.groups groups, then group i's
// secondary scores over its B = E / A experts at A + i*B.  `fetch(c, l, z)` fills
// l[0..15] with the scores of columns c .. c+15 (c a multiple of 16).
//   pass 1  top-(k_primary+1) of the primary scores (TopList, ties to the lower group)
//   pass 2  every secondary column once, in ascending order; a column of one of this
//           token's chosen groups enters that group's top-(k_group+1) list
//   gates   Softmax(KeepTopK) at each level, multiplied; expert j of group i is i*B + j
// Everything stays in registers: no shared memory and no barrier.
template <int KP, int KG, class Fetch>
__device__ __forceinline__ void gate_tile_hier(const Fetch& fetch, int q, int lane, int64_t tile,
                                               const GateArgs& g) {
  const int row = q * 32 + lane;
  const int64_t t = tile * 128 + row;
  const bool valid = t < g.T;
  const int A = g.groups, NG = g.groups + g.E, B = g.E / g.groups;
  const int k1 = g.k_primary, k2 = g.k / g.k_primary;
  TopList<KP> prim;
  prim.init();
#pragma unroll 1
  for (int cs = 0; cs < A; cs += 16) {
    float l[16], z[16];
    fetch(cs, l, z);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (cs + j < A) prim.push(l[j], cs + j);
  }
  int chosen[KP];
#pragma unroll
  for (int q2 = 0; q2 < KP; ++q2) chosen[q2] = (q2 < k1) ? prim.i[q2] : -1;
  TopList<KG> sec[KP];
#pragma unroll
  for (int q2 = 0; q2 < KP; ++q2) sec[q2].init();
  // (grp, e): group and expert-in-group of column c, advanced column by column
  int grp = 0, e = 0;
#pragma unroll 1
  for (int cs = (A / 16) * 16; cs < NG; cs += 16) {
    float l[16], z[16];
    fetch(cs, l, z);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = cs + j;
      if (c >= A && c < NG) {
#pragma unroll
        for (int q2 = 0; q2 < KP; ++q2)
          if (chosen[q2] == grp) sec[q2].push(l[j], e);
        if (++e == B) {
          e = 0;
          ++grp;
        }
      }
    }
  }
  // primary gates over the kept groups, and the primary k-th vs (k+1)-th gap
  float gp[KP];
  float den = 0.0f;
#pragma unroll
  for (int q2 = 0; q2 < KP; ++q2) {
    gp[q2] = (q2 < k1) ? expf(prim.v[q2] - prim.v[0]) : 0.0f;
    den += gp[q2];
  }
  float kth = INFINITY, kth1 = -INFINITY;
#pragma unroll
  for (int j = 0; j <= KP; ++j) {
    if (j < k1) kth = fminf(kth, prim.v[j]);
    else kth1 = fmaxf(kth1, prim.v[j]);
  }
  float gap = (k1 < A) ? kth - kth1 : INFINITY;
#pragma unroll
  for (int q2 = 0; q2 < KP; ++q2) {
    if (q2 >= k1) continue;
    const float share = gp[q2] / den;
    float gs[KG];
    float ds = 0.0f;
#pragma unroll
    for (int j = 0; j < KG; ++j) {
      gs[j] = (j < k2) ? expf(sec[q2].v[j] - sec[q2].v[0]) : 0.0f;
      ds += gs[j];
    }
    float sk = INFINITY, sk1 = -INFINITY;
#pragma unroll
    for (int j = 0; j <= KG; ++j) {
      if (j < k2) sk = fminf(sk, sec[q2].v[j]);
      else sk1 = fmaxf(sk1, sec[q2].v[j]);
    }
    if (k2 < B) gap = fminf(gap, sk - sk1);
    if (valid) {
#pragma unroll
      for (int j = 0; j < KG; ++j)
        if (j < k2) {
          g.topk_idx[t * g.k + q2 * k2 + j] = chosen[q2] * B + sec[q2].i[j];
          g.topk_gate[t * g.k + q2 * k2 + j] = share * (gs[j] / ds);
        }
    }
  }
  if (valid && g.near_tie) g.near_tie[t] = (gap <= 1e-4f) ? 1 : 0;
}

// The hierarchical gate of the tensor-core router, spread over column groups: the same
// token rows and score columns as gate_tile_hier, with the thread in lane l of gate warp
// w owning row r = 32*q + l of column group grp = w / 4 (with half tiles, 64 tokens in
// both halves of the MMA operand: row 32*(q & 1) + l of column group 2*grp + q / 2, as
// in gate_tile).  Every thread scores the primary columns of its token; column group cg
// then forms the secondary list of each group i = cg, cg + CG, ... over that group's
// columns in ascending order (a fresh list per group, so no thread walks the groups it
// does not own) and, where its token kept group i, writes that group's assignments.
// Results equal gate_tile_hier's: the same lists, gates and gaps, formed by the same
// operations.  The per-token minimum gap over the kept groups meets in shared memory.
template <int KP, int KG, int G, class Fetch, class Sync>
__device__ __forceinline__ void gate_tile_hier_cg(const Fetch& fetch, const Sync& sync, int q,
                                                  int grp, int lane, int64_t tile, bool half,
                                                  const GateArgs& g, uint8_t* smem) {
  const int ntok = half ? 64 : 128;
  const int row = half ? (q & 1) * 32 + lane : q * 32 + lane;
  const int CG = half ? 2 * G : G;
  const int cgrp = half ? grp * 2 + (q >> 1) : grp;
  const int64_t t = tile * ntok + row;
  const bool valid = t < g.T;
  const int A = g.groups, B = g.E / g.groups;
  const int k1 = g.k_primary, k2 = g.k / g.k_primary;
  TopList<KP> prim;
  prim.init();
#pragma unroll 1
  for (int cs = 0; cs < A; cs += 16) {
    float l[16], z[16];
    fetch(cs, l, z);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (cs + j < A) prim.push(l[j], cs + j);
  }
  float gp[KP];
  float den = 0.0f;
#pragma unroll
  for (int q2 = 0; q2 < KP; ++q2) {
    gp[q2] = (q2 < k1) ? expf(prim.v[q2] - prim.v[0]) : 0.0f;
    den += gp[q2];
  }
  float gmin = INFINITY;  // smallest secondary gap over the kept groups this thread owns
#pragma unroll 1
  for (int i = cgrp; i < A; i += CG) {
    TopList<KG> cur;
    cur.init();
    const int c0 = A + i * B, c1 = c0 + B;
#pragma unroll 1
    for (int cs = c0 & ~15; cs < c1; cs += 16) {
      float l[16], z[16];
      fetch(cs, l, z);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (cs + j >= c0 && cs + j < c1) cur.push(l[j], cs + j - c0);
    }
    // the rank of group i among this token's kept groups, if it kept it
    int slot = -1;
    float share = 0.0f;
#pragma unroll
    for (int q2 = 0; q2 < KP; ++q2)
      if (q2 < k1 && prim.i[q2] == i) {
        slot = q2;
        share = gp[q2] / den;
      }
    if (slot >= 0) {
      float gs[KG];
      float ds = 0.0f;
#pragma unroll
      for (int j = 0; j < KG; ++j) {
        gs[j] = (j < k2) ? expf(cur.v[j] - cur.v[0]) : 0.0f;
        ds += gs[j];
      }
      float sk = INFINITY, sk1 = -INFINITY;
#pragma unroll
      for (int j = 0; j <= KG; ++j) {
        if (j < k2) sk = fminf(sk, cur.v[j]);
        else sk1 = fmaxf(sk1, cur.v[j]);
      }
      if (k2 < B) gmin = fminf(gmin, sk - sk1);
      if (valid) {
#pragma unroll
        for (int j = 0; j < KG; ++j)
          if (j < k2) {
            g.topk_idx[t * g.k + slot * k2 + j] = i * B + cur.i[j];
            g.topk_gate[t * g.k + slot * k2 + j] = share * (gs[j] / ds);
          }
      }
    }
  }
  if (g.near_tie != nullptr) {  // uniform across the gate threads
    float* hg = reinterpret_cast<float*>(smem);  // [CG][ntok]
    hg[cgrp * ntok + row] = gmin;
    sync();
    if (cgrp == 0 && valid) {
      float kth = INFINITY, kth1 = -INFINITY;
#pragma unroll
      for (int j = 0; j <= KP; ++j) {
        if (j < k1) kth = fminf(kth, prim.v[j]);
        else kth1 = fmaxf(kth1, prim.v[j]);
      }
      float gap = (k1 < A) ? kth - kth1 : INFINITY;
      for (int c2 = 0; c2 < CG; ++c2) gap = fminf(gap, hg[c2 * ntok + row]);
      g.near_tie[t] = (gap <= 1e-4f) ? 1 : 0;
    }
  }
}

// ------------------------------------------------------------------ bf16 router
//
// Persistent and warp-specialised.  Warp 0 streams the x tile and the gating weights of
// each of the CTA's token tiles through a ring of shared-memory stages (TMA); warp 1
// issues the MMAs of a tile into one of two TMEM accumulator buffers (one when the two
// products of noisy gating fill TMEM); the 4*G gate warps read a finished buffer, run
// the gate and hand the buffer back.  So one tile's gate overlaps the next tile's loads
// and MMAs.

namespace rt {
// expert-column groups per token: 4 (16 gate warps), or 2 for k > 4 to leave registers
// for the longer top-(k+1) lists
constexpr int groups_for(int KM) { return KM > 4 ? 2 : 4; }
constexpr int BK = 64;
constexpr int A_BYTES = kRouteBM * BK * 2;  // 16 KB
constexpr int GATE_WARP0 = 2;
}  // namespace rt

struct RouteTcArgs {
  GateArgs g;
  int e_pad;      // E rounded up to a multiple of 16 (the MMA N)
  int acc_cols;   // TMEM columns per accumulator (power of two >= 32, >= e_pad)
  int kblocks;    // d / 64
  int nb;         // 1, or 2 with W_noise
  int nbuf;       // TMEM accumulator buffers: 2, or 1 when 2 * nb * acc_cols > 512
  int stages;
  int half;       // 1: 64-token tiles, each loaded into both halves of the MMA operand
  int ntiles;     // ceil(T / 128), or ceil(T / 64) with half tiles
  int gate_off;   // byte offset of the gate scratch in shared memory
  int bar_off;    // byte offset of the barriers
  int* err;
};

__device__ __forceinline__ void gate_bar_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// HKG > 0: hierarchical gating with KM the primary and HKG the secondary list bucket.
template <int KM, int HKG = 0, int G = rt::groups_for(KM)>
__global__ void __launch_bounds__(64 + 128 * G)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmG,
                    const __grid_constant__ CUtensorMap tmN, const RouteTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int b_bytes = a.e_pad * rt::BK * 2;
  const int stage_bytes = rt::A_BYTES + a.nb * b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + a.stages);
  const uint32_t tfull0 = smem_u32(bars + 2 * a.stages);
  const uint32_t tempty0 = smem_u32(bars + 2 * a.stages + 2);
  const uint32_t drain = smem_u32(bars + 2 * a.stages + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * a.stages + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* s_gate_fail = reinterpret_cast<volatile int*>(tmem_holder + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t buf_cols = static_cast<uint32_t>(a.nb * a.acc_cols);
  const uint32_t ncols = buf_cols * static_cast<uint32_t>(a.nbuf);
  constexpr int GATE_WARPS = 4 * G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, GATE_WARPS);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_gate_fail = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmG);
    if (a.nb == 2) tma_prefetch_desc(&tmN);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  grid_dep_wait();  // x, and readers of the outputs, belong to earlier kernels
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool aborted = false;
      for (int L = blockIdx.x; L < a.ntiles && !aborted; L += gridDim.x) {
        for (int kb = 0; kb < a.kblocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, s_abort)) {
            aborted = true;
            break;
          }
          uint8_t* st = smem + stage * stage_bytes;
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, static_cast<uint32_t>(stage_bytes));
          if (a.half) {  // the same 64 token rows into operand rows 0-63 and 64-127
            tma_load_2d(smem_u32(st), &tmX, fb, kb * rt::BK, L * 64);
            tma_load_2d(smem_u32(st + rt::A_BYTES / 2), &tmX, fb, kb * rt::BK, L * 64);
          } else {
            tma_load_2d(smem_u32(st), &tmX, fb, kb * rt::BK, L * kRouteBM);
          }
          tma_load_2d(smem_u32(st + rt::A_BYTES), &tmG, fb, kb * rt::BK, 0);
          if (a.nb == 2) tma_load_2d(smem_u32(st + rt::A_BYTES + b_bytes), &tmN, fb, kb * rt::BK, 0);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        // let every copy this thread started land before the CTA releases its smem
        for (int s = 0; s < a.stages; ++s)
          if (armed & (1u << s)) mbar_wait(full0 + 8 * s, (armed_par >> s) & 1, nullptr, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_f32acc(kRouteBM, a.e_pad, kFmtBF16);
      int stage = 0, buf = 0;
      uint32_t phase = 0, buf_phase = 0;
      bool aborted = false;
      for (int L = blockIdx.x; L < a.ntiles && !aborted; L += gridDim.x) {
        if (!mbar_wait(tempty0 + 8 * buf, buf_phase ^ 1, s_abort)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf) * buf_cols;
        for (int kb = 0; kb < a.kblocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, s_abort)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * stage_bytes);
#pragma unroll
          for (int kk = 0; kk < rt::BK / 16; ++kk) {
            const uint64_t ad = sdesc_k128(st + kk * 32);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_f16kind(d0, ad, sdesc_k128(st + rt::A_BYTES + kk * 32), idesc, acc);
            if (a.nb == 2)
              tc_mma_f16kind(d0 + a.acc_cols, ad,
                             sdesc_k128(st + rt::A_BYTES + b_bytes + kk * 32), idesc, acc);
          }
          tc_commit(empty0 + 8 * stage);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        tc_commit(tfull0 + 8 * buf);
        if (++buf == a.nbuf) {
          buf = 0;
          buf_phase ^= 1;
        }
      }
      if (aborted) {
        set_error(a.err, kErrTimeout);
        *s_abort = 1;
        tc_commit(drain);  // wait for the MMAs already issued before TMEM is freed
        mbar_wait(drain, 0, nullptr, kDrainLimitNs);
      }
    }
  } else {
    // -------------------------------------------------------------- gate warps
    const int gw = warp - rt::GATE_WARP0;  // 0 .. 4G-1
    const int q = warp & 3;                // TMEM lane quarter this warp may read
    const int grp = gw >> 2;
    const int gtid = gw * 32 + lane;
    auto sync = [] { gate_bar_sync(128 * G); };
    uint8_t* gsm = smem + a.gate_off;
    load_bias_smem(a.g, gsm, KM, G, gtid, 128 * G);
    sync();
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int L = blockIdx.x; L < a.ntiles; L += gridDim.x) {
      // every gate warp waits; the decision to stop is taken together after a barrier,
      // so that no gate warp is left at one of the gate's barriers
      if (!mbar_wait(tfull0 + 8 * buf, buf_phase, s_abort)) *s_gate_fail = 1;
      sync();
      if (*s_gate_fail) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(buf) * buf_cols;
      if (a.nb == 2) {
        // noisy gating: 16 columns of x.W_g and of x.W_noise per wait
        auto fetch = [&](int c, float (&l)[16], float (&z)[16]) {
          uint32_t v[16], w[16];
          tmem_ld16(tmem_base + lane_base + c, v);
          tmem_ld16(tmem_base + lane_base + a.acc_cols + c, w);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            l[j] = __uint_as_float(v[j]);
            z[j] = __uint_as_float(w[j]);
          }
        };
        gate_tile<KM, G, 16>(fetch, sync, q, grp, gtid, L, a.half != 0, a.g, gsm);
      } else {
        auto fetch = [&](int c, float (&l)[16], float (&z)[16]) {
          uint32_t v[16];
          tmem_ld16(tmem_base + lane_base + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            l[j] = __uint_as_float(v[j]);
            z[j] = 0.0f;
          }
        };
        if constexpr (HKG > 0) {
          gate_tile_hier_cg<KM, HKG, G>(fetch, sync, q, grp, lane, L, a.half != 0, a.g, gsm);
        } else {
          gate_tile<KM, G, 16>(fetch, sync, q, grp, gtid, L, a.half != 0, a.g, gsm);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
      if (++buf == a.nbuf) {
        buf = 0;
        buf_phase ^= 1;
      }
    }
    if (*s_gate_fail && gtid == 0) set_error(a.err, kErrTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, ncols);
}

// ------------------------------------------------------------------ fp32 router

// The logits were written to the workspace by the SIMT product; 128 threads, one token
// row each, walk all expert columns (one column group).
template <int KM>
__global__ void __launch_bounds__(128, 1)
    gate_f32_kernel(const float* __restrict__ logits, const float* __restrict__ nz, GateArgs g) {
  extern __shared__ __align__(16) uint8_t gsmem[];
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteBM;
  const int64_t t = t0 + threadIdx.x;
  const bool valid = t < g.T;
  const int E = g.E;
  auto fetch = [&](int c, float (&l)[16], float (&z)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const bool in = valid && (c + j < E);
      l[j] = in ? logits[t * E + c + j] : 0.0f;
      z[j] = (in && nz != nullptr) ? nz[t * E + c + j] : 0.0f;
    }
  };
  const int warp = threadIdx.x >> 5;
  load_bias_smem(g, gsmem, KM, 1, static_cast<int>(threadIdx.x), 128);
  __syncthreads();
  gate_tile<KM, 1, 16>(fetch, [] { __syncthreads(); }, warp, 0, static_cast<int>(threadIdx.x),
                       static_cast<int64_t>(blockIdx.x), false, g, gsmem);
}

// Hierarchical gate on the fp32 logits [T, groups + E] of the workspace: 128 threads,
// one token row each.
template <int KP, int KG>
__global__ void __launch_bounds__(128, 1)
    gate_f32_hier_kernel(const float* __restrict__ logits, GateArgs g) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteBM + threadIdx.x;
  const bool valid = t < g.T;
  const int NG = g.groups + g.E;
  auto fetch = [&](int c, float (&l)[16], float (&z)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const bool in = valid && (c + j < NG);
      l[j] = in ? logits[t * NG + c + j] : 0.0f;
      z[j] = 0.0f;
    }
  };
  gate_tile_hier<KP, KG>(fetch, static_cast<int>(threadIdx.x) >> 5,
                         static_cast<int>(threadIdx.x) & 31, static_cast<int64_t>(blockIdx.x), g);
}

// Importance and Load partial sums of noisy gating from the gate's per-token values.
// Block (chunk, slice) covers a run of tokens and 8*R experts; warp w of the block takes
// experts slice*8R + w*R .. +R-1 and its lanes the run's tokens 32 at a time, each lane
// reading its token's chosen experts, gates and k-th / (k+1)-th scores once and then the
// warp's R experts' values (a warp reads 128 contiguous bytes per expert and quantity).
// For token t and expert e:
//   Importance term: the gate of e if e is one of t's chosen experts, else 0
//   Load term: P(t, e) = Phi((l_te - kth_excluding(H_t, k, e)) / Softplus(z_te)), where
//   kth_excluding is the (k+1)-th largest score when H_te >= the k-th largest, else the
//   k-th largest (H_te as the gate formed it, so H >= the k-th means "among the top k").
// Each lane adds its tokens in increasing order, then the lanes of each expert column are
// summed in a fixed butterfly order into partials[chunk][2][E], so the result does not
// depend on scheduling.
template <int R>
__global__ void __launch_bounds__(256)
    importance_load_kernel(const float* __restrict__ lw, const float* __restrict__ sw,
                           const float* __restrict__ hw, const float* __restrict__ kw,
                           const int32_t* __restrict__ topk_idx,
                           const float* __restrict__ topk_gate, int64_t T, int E, int k,
                           int64_t chunk_tokens, int want_load, float* __restrict__ partials) {
  static_assert(R % 8 == 0, "experts per warp: whole 8-column reduce steps");
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = (blockIdx.y * 8 + warp) * R;
  if (e0 >= E) return;  // the whole warp
  const int64_t t_lo = static_cast<int64_t>(blockIdx.x) * chunk_tokens;
  const int64_t t_hi = min(T, t_lo + chunk_tokens);
  float si[R], sl[R];
#pragma unroll
  for (int r = 0; r < R; ++r) si[r] = sl[r] = 0.0f;
  for (int64_t tb = t_lo; tb < t_hi; tb += 32) {
    const int64_t t = tb + lane;
    const bool tv = t < t_hi;
    int id[8];
    float gv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = tv && j < k;
      id[j] = in ? __ldg(topk_idx + t * k + j) : -1;
      gv[j] = in ? __ldg(topk_gate + t * k + j) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = e0 + r;
      float gi = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) gi = (id[j] == e) ? gv[j] : gi;
      si[r] += gi;
    }
    if (want_load) {  // uniform over the grid
      // every load of the group first (a lane past the run or an expert past E reads an
      // in-range element and discards it), then the arithmetic: the kernel is bound by
      // load latency, not by bytes
      const int64_t tt = tv ? t : t_hi - 1;
      const float k0 = __ldg(kw + tt), k1 = __ldg(kw + T + tt);
      float li[R], sp[R], H[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t i = static_cast<int64_t>(min(e0 + r, E - 1)) * T + tt;
        li[r] = __ldg(lw + i);
        sp[r] = __ldg(sw + i);
        H[r] = __ldg(hw + i);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float ex = (H[r] >= k0) ? k1 : k0;
        const float pl = 0.5f + 0.5f * erf_as7126(__fdividef(li[r] - ex, sp[r]) * 0.70710678118654752f);
        sl[r] += (tv && e0 + r < E) ? pl : 0.0f;
      }
    }
  }
  // column sums over the lanes, 8 experts at a time
#pragma unroll
  for (int g8 = 0; g8 < R / 8; ++g8) {
    float a8[8], b8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      a8[j] = si[8 * g8 + j];
      b8[j] = sl[8 * g8 + j];
    }
    const float ci = warp_colsum8(a8, lane);
    const float cl = warp_colsum8(b8, lane);
    const int e = e0 + 8 * g8 + colsum8_column(lane);
    if (lane < 8 && e < E) {
      partials[(blockIdx.x * 2 + 0) * static_cast<int64_t>(E) + e] = ci;
      partials[(blockIdx.x * 2 + 1) * static_cast<int64_t>(E) + e] = cl;
    }
  }
}

// Importance[e] (blockIdx.y = 0) and Load[e] (blockIdx.y = 1) from the per-block
// partials [nblocks][2][E]: one block per expert and quantity, each thread a fixed strided
// subset of the partials in order, then a fixed tree over the block, so the sum is the
// same on every run.
__global__ void __launch_bounds__(256)
    finalize_importance_load_kernel(const float* __restrict__ partials, int nblocks, int E,
                                    float* importance, float* load) {
  const int e = blockIdx.x, which = blockIdx.y;
  grid_dep_wait();
  grid_dep_launch();
  float* out = which == 0 ? importance : load;
  if (out == nullptr) return;  // uniform over the block
  float s = 0.0f;
  for (int b = threadIdx.x; b < nblocks; b += 256)
    s += partials[(static_cast<int64_t>(b) * 2 + which) * E + e];
  s = block_sum_fixed<256>(s);
  if (threadIdx.x == 0) out[e] = s;
}

// ------------------------------------------------------------------ launchers

static GateArgs gate_args(const RouteProblem& p) {
  GateArgs g;
  g.T = p.T;
  g.E = p.E;
  g.k = p.k;
  g.noisy = p.noisy;
  g.renorm = p.renorm;
  g.groups = p.hier ? p.groups : 0;
  g.k_primary = p.hier ? p.k_primary : 0;
  g.noise = p.noise;
  g.bias = p.bias;
  g.topk_idx = p.topk_idx;
  g.topk_gate = p.topk_gate;
  g.near_tie = p.near_tie;
  g.partials = (p.importance || p.load) ? p.partials : nullptr;
  g.lw = g.sw = g.hw = g.kw = nullptr;
  g.split = 0;
  return g;
}

static int k_bucket(int k) { return k <= 1 ? 1 : k <= 2 ? 2 : k <= 4 ? 4 : 8; }

static cudaError_t launch_finalize(const RouteProblem& p, int nblocks, const LaunchCtx& c) {
  if (!(p.importance || p.load)) return cudaSuccess;
  return launch_kernel(finalize_importance_load_kernel, dim3(p.E, 2), dim3(256), 0, c,
                       static_cast<const float*>(p.partials), nblocks, p.E, p.importance, p.load);
}

template <int KM, int HKG = 0>
static cudaError_t launch_route_tc(const CUtensorMap& tmX, const CUtensorMap& tmG,
                                   const CUtensorMap& tmN, const RouteTcArgs& a, int smem,
                                   int grid, const LaunchCtx& c) {
  cudaError_t e = ensure_smem_limit(route_tc_kernel<KM, HKG>, smem);
  if (e != cudaSuccess) return e;
  const int G = rt::groups_for(KM);
  return launch_kernel(route_tc_kernel<KM, HKG>, dim3(grid), dim3(64 + 128 * G), smem, c, tmX, tmG,
                       tmN, a);
}

// hierarchical: list buckets of the primary (KP) and secondary (KG) levels, 1, 2 or 4
template <int KP>
static cudaError_t launch_route_tc_hier(int kg, const CUtensorMap& tmX, const CUtensorMap& tmG,
                                        const RouteTcArgs& a, int smem, int grid,
                                        const LaunchCtx& c) {
  switch (kg) {
    case 1: return launch_route_tc<KP, 1>(tmX, tmG, tmG, a, smem, grid, c);
    case 2: return launch_route_tc<KP, 2>(tmX, tmG, tmG, a, smem, grid, c);
    default: return launch_route_tc<KP, 4>(tmX, tmG, tmG, a, smem, grid, c);
  }
}

// Noisy gating on the tensor-core path with Importance or Load asked for: after the
// router kernel, the sums over the whole grid (importance_load_kernel), then the fixed-
// order total over the chunks.
template <int R>
static cudaError_t launch_importance_load_r(const RouteProblem& p, int64_t chunks, int64_t per,
                                           const LaunchCtx& c) {
  const int slices = (p.E + 8 * R - 1) / (8 * R);
  return launch_kernel(importance_load_kernel<R>, dim3(static_cast<unsigned>(chunks), slices),
                       dim3(256), 0, c, static_cast<const float*>(p.lw),
                       static_cast<const float*>(p.sw), static_cast<const float*>(p.hw),
                       static_cast<const float*>(p.kw), static_cast<const int32_t*>(p.topk_idx),
                       static_cast<const float*>(p.topk_gate), p.T, p.E, p.k, per,
                       p.load != nullptr ? 1 : 0, p.partials);
}

static cudaError_t launch_importance_load(const RouteProblem& p, const LaunchCtx& c) {
  // experts per warp: a block's eight warps cover up to 8R experts
  const int R = p.E <= 64 ? 8 : 16;
  const int slices = (p.E + 8 * R - 1) / (8 * R);
  // token runs of whole 32-token groups, about two blocks per SM, at most one run per
  // 64 tokens (the partials' rows)
  int64_t chunks = (2LL * c.num_sms + slices - 1) / slices;
  const int64_t cap = route_blocks(p.T);
  if (chunks > cap) chunks = cap;
  if (chunks < 1) chunks = 1;
  int64_t per = (p.T + chunks - 1) / chunks;
  per = per < 32 ? 32 : (per + 31) / 32 * 32;
  chunks = (p.T + per - 1) / per;
  cudaError_t e = R == 8 ? launch_importance_load_r<8>(p, chunks, per, c)
                         : launch_importance_load_r<16>(p, chunks, per, c);
  if (e != cudaSuccess) return e;
  return launch_kernel(finalize_importance_load_kernel, dim3(p.E, 2), dim3(256), 0, c,
                       static_cast<const float*>(p.partials), static_cast<int>(chunks), p.E,
                       p.importance, p.load);
}

cudaError_t launch_route_bf16(const RouteProblem& p, const LaunchCtx& c) {
  RouteTcArgs a;
  a.g = gate_args(p);
  const bool split = p.noisy && (p.importance || p.load) && p.lw != nullptr;
  if (split || p.store_scores) {
    a.g.lw = p.lw;
    if (p.noisy) {
      a.g.sw = p.sw;
      a.g.hw = p.hw;
      a.g.kw = p.kw;
    }
  }
  a.g.split = split ? 1 : 0;
  const int n_scores = p.hier ? p.E + p.groups : p.E;  // score columns (rows of w_gate)
  a.e_pad = (n_scores + 15) / 16 * 16;
  a.acc_cols = 32;
  while (a.acc_cols < a.e_pad) a.acc_cols <<= 1;
  a.kblocks = p.d / rt::BK;
  a.nb = p.noisy ? 2 : 1;
  a.nbuf = 2 * a.nb * a.acc_cols <= 512 ? 2 : 1;
  // half tiles when 128-token tiles would fill at most half of the SMs
  const int full_tiles = static_cast<int>((p.T + kRouteBM - 1) / kRouteBM);
  a.half = (2 * full_tiles <= c.num_sms) ? 1 : 0;
  a.ntiles = a.half ? static_cast<int>((p.T + 63) / 64) : full_tiles;
  const int km = p.hier ? k_bucket(p.k_primary) : k_bucket(p.k);
  const int scratch = gate_smem_bytes(km, rt::groups_for(km), p.E);
  const int stage_bytes = rt::A_BYTES + a.nb * a.e_pad * rt::BK * 2;
  // the ring takes what the gate scratch and the barriers leave of 227 KB
  const int bar_bytes = 8 * (2 * 8 + 5) + 16;
  int stages = (227 * 1024 - 1024 - (scratch + 127) / 128 * 128 - bar_bytes) / stage_bytes;
  if (stages > 8) stages = 8;
  if (stages < 2) return cudaErrorInvalidValue;  // not reached for E <= 256, d % 64 == 0
  a.stages = stages;
  a.gate_off = stages * stage_bytes;
  a.bar_off = a.gate_off + (scratch + 127) / 128 * 128;
  a.err = c.err;
  const int smem = 1024 + a.bar_off + 8 * (2 * stages + 5) + 16;

  CUtensorMap tmX, tmG, tmN;
  if (!make_tmap_bf16(&tmX, p.x, static_cast<uint64_t>(p.T), p.d, a.half ? 64 : kRouteBM))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tmG, p.w_gate, static_cast<uint64_t>(n_scores), p.d, a.e_pad))
    return cudaErrorInvalidValue;
  if (p.noisy) {
    if (!make_tmap_bf16(&tmN, p.w_noise, static_cast<uint64_t>(p.E), p.d, a.e_pad)) return cudaErrorInvalidValue;
  } else {
    tmN = tmG;
  }
  const int grid = a.ntiles < c.num_sms ? a.ntiles : c.num_sms;
  cudaError_t e;
  if (p.hier) {
    const int kg = k_bucket(p.k / p.k_primary);
    switch (km) {
      case 1: e = launch_route_tc_hier<1>(kg, tmX, tmG, a, smem, grid, c); break;
      case 2: e = launch_route_tc_hier<2>(kg, tmX, tmG, a, smem, grid, c); break;
      default: e = launch_route_tc_hier<4>(kg, tmX, tmG, a, smem, grid, c); break;
    }
    return e;
  }
  switch (km) {
    case 1: e = launch_route_tc<1>(tmX, tmG, tmN, a, smem, grid, c); break;
    case 2: e = launch_route_tc<2>(tmX, tmG, tmN, a, smem, grid, c); break;
    case 4: e = launch_route_tc<4>(tmX, tmG, tmN, a, smem, grid, c); break;
    default: e = launch_route_tc<8>(tmX, tmG, tmN, a, smem, grid, c); break;
  }
  if (e != cudaSuccess) return e;
  if (split) return launch_importance_load(p, c);
  return launch_finalize(p, a.ntiles, c);
}

template <int KM>
static cudaError_t launch_gate_f32(const RouteProblem& p, const GateArgs& g, int nblocks,
                                   const LaunchCtx& c) {
  const int smem = gate_smem_bytes(KM, 1, p.E);
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_smem_limit(gate_f32_kernel<KM>, smem);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(gate_f32_kernel<KM>, dim3(nblocks), dim3(128), smem, c,
                       static_cast<const float*>(p.logits_ws),
                       static_cast<const float*>(p.noisy ? p.nz_ws : nullptr), g);
}

template <int KP>
static cudaError_t launch_gate_f32_hier(int kg, const RouteProblem& p, const GateArgs& g,
                                        int nblocks, const LaunchCtx& c) {
  const float* lg = p.logits_ws;
  switch (kg) {
    case 1: return launch_kernel(gate_f32_hier_kernel<KP, 1>, dim3(nblocks), dim3(128), 0, c, lg, g);
    case 2: return launch_kernel(gate_f32_hier_kernel<KP, 2>, dim3(nblocks), dim3(128), 0, c, lg, g);
    default: return launch_kernel(gate_f32_hier_kernel<KP, 4>, dim3(nblocks), dim3(128), 0, c, lg, g);
  }
}

cudaError_t launch_route_f32(const RouteProblem& p, const LaunchCtx& c) {
  const int n_scores = p.hier ? p.E + p.groups : p.E;
  cudaError_t e = launch_sgemm_grouped(static_cast<const float*>(p.x), static_cast<const float*>(p.w_gate),
                                       p.logits_ws, nullptr, 1, p.T, n_scores, p.d, 0, c);
  if (e != cudaSuccess) return e;
  if (p.hier) {
    const GateArgs g = gate_args(p);
    const int nblocks = static_cast<int>((p.T + kRouteBM - 1) / kRouteBM);
    const int kg = k_bucket(p.k / p.k_primary);
    switch (k_bucket(p.k_primary)) {
      case 1: return launch_gate_f32_hier<1>(kg, p, g, nblocks, c);
      case 2: return launch_gate_f32_hier<2>(kg, p, g, nblocks, c);
      default: return launch_gate_f32_hier<4>(kg, p, g, nblocks, c);
    }
  }
  if (p.noisy) {
    e = launch_sgemm_grouped(static_cast<const float*>(p.x), static_cast<const float*>(p.w_noise),
                             p.nz_ws, nullptr, 1, p.T, p.E, p.d, 0, c);
    if (e != cudaSuccess) return e;
  }
  const GateArgs g = gate_args(p);
  const int nblocks = static_cast<int>((p.T + kRouteBM - 1) / kRouteBM);
  switch (k_bucket(p.k)) {
    case 1: e = launch_gate_f32<1>(p, g, nblocks, c); break;
    case 2: e = launch_gate_f32<2>(p, g, nblocks, c); break;
    case 4: e = launch_gate_f32<4>(p, g, nblocks, c); break;
    default: e = launch_gate_f32<8>(p, g, nblocks, c); break;
  }
  if (e != cudaSuccess) return e;
  return launch_finalize(p, nblocks, c);
}

}  // namespace moe
