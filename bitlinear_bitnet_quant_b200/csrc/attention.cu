// Attention core of the stacked layer: rotary position embedding, the key /
// value cache, and causal softmax attention.
//
// "AI 혁신의 선두: 마이크로소프트의 1비트 LLM, BitNet b1.58 2B4T", section 주요
// 아키텍처 혁신: the model uses rotary position embedding; its linear layers
// (the Q/K/V/O projections around this core) are BitLinear.  The pages give
// no formula, so the rotary embedding's own definition is used: in each head
// of width d, the pair (x[2i], x[2i+1]) of a token at position p turns by the
// angle p * theta_i, theta_i = base^(-2i/d).  Attention is, per head,
// softmax(q k^T / sqrt(d)) v over the keys at positions up to the query's.
//
// Layout: token rows [B * L][heads * d] fp32, sequence b's tokens l = 0..L-1
// at positions t0 + l; caches Kc, Vc [B][T_cap][heads * d] fp32 (rotated keys,
// values), row t = position t.
//
// Precision: the rotation is computed in fp64 (angle, cosine and sine, the
// two products and their sum) and rounded once to fp32.  Attention runs in
// fp32 on the CUDA cores (fused multiply-adds, expf), with the running-max
// rescaling of the softmax (max, sum and output updated key block by key
// block, which is exact in real arithmetic).  No integer code is decided
// here, so results are compared with a float64 evaluation within the bound
// the fp32 arithmetic allows.
#include "common.cuh"

namespace bitnet {

constexpr int ATT_D = 128;                         // head width

// ---------------------------------------------------------------------------
// rotary embedding of Q (in place) and K (into the cache), V into the cache
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
rope_append_kernel(float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V, int B, int L,
                   int t0, int HD, int d, double log2_base, float* __restrict__ Kc, float* __restrict__ Vc,
                   int T_cap) {
  pdl_launch_dependents();
  pdl_wait();                                      // Q, K and V come from the previous kernel
  const int pairs = HD / 2;
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (size_t)B * L * pairs) return;
  const int r = (int)(idx / pairs);                // token row
  const int pr = (int)(idx - (size_t)r * pairs);   // pair inside the row
  const int b = r / L, l = r - b * L;
  const int pos = t0 + l;
  const int i = pr % (d / 2);                      // pair inside the head
  const double theta = exp2(-(2.0 * i / d) * log2_base);
  double sn, cs;
  sincos((double)pos * theta, &sn, &cs);
  const size_t off = (size_t)r * HD + 2 * (size_t)pr;
  const size_t coff = ((size_t)b * T_cap + pos) * HD + 2 * (size_t)pr;
  const float2 q = *reinterpret_cast<const float2*>(Q + off);
  const float2 k = *reinterpret_cast<const float2*>(K + off);
  const float2 v = *reinterpret_cast<const float2*>(V + off);
  *reinterpret_cast<float2*>(Q + off) =
      make_float2((float)((double)q.x * cs - (double)q.y * sn), (float)((double)q.x * sn + (double)q.y * cs));
  *reinterpret_cast<float2*>(Kc + coff) =
      make_float2((float)((double)k.x * cs - (double)k.y * sn), (float)((double)k.x * sn + (double)k.y * cs));
  *reinterpret_cast<float2*>(Vc + coff) = v;
}

// ---------------------------------------------------------------------------
// few queries per sequence (decode): one CTA per (token, head); its 8 warps
// take every eighth key of the context, each with its own running max, sum
// and output; the warps' partial softmaxes are merged at the end.  A lane
// holds 4 of the head's 128 dimensions.
// ---------------------------------------------------------------------------
constexpr int ATD_WARPS = 8;
constexpr int ATD_UNROLL = 4;

__global__ void __launch_bounds__(32 * ATD_WARPS)
attention_decode_kernel(const float* __restrict__ Q, const float* __restrict__ Kc, const float* __restrict__ Vc,
                        int L, int t0, int HD, int T_cap, float scale, float* __restrict__ A) {
  __shared__ float sm_m[ATD_WARPS], sm_l[ATD_WARPS];
  __shared__ float4 sm_o[ATD_WARPS][32];
  pdl_launch_dependents();
  pdl_wait();                                      // Q and the caches come from the previous kernel
  const int r = blockIdx.x, h = blockIdx.y;
  const int b = r / L, l = r - b * L;
  const int n = t0 + l + 1;                        // keys visible to this query
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4 q = *reinterpret_cast<const float4*>(Q + (size_t)r * HD + h * ATT_D + 4 * lane);
  const float* kb = Kc + (size_t)b * T_cap * HD + h * ATT_D + 4 * lane;
  const float* vb = Vc + (size_t)b * T_cap * HD + h * ATT_D + 4 * lane;
  float m = -INFINITY, sum = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = warp * ATD_UNROLL; j0 < n; j0 += ATD_WARPS * ATD_UNROLL) {
    float4 kv[ATD_UNROLL], vv[ATD_UNROLL];
#pragma unroll
    for (int u = 0; u < ATD_UNROLL; ++u) {
      const int j = j0 + u < n ? j0 + u : n - 1;
      kv[u] = *reinterpret_cast<const float4*>(kb + (size_t)j * HD);
      vv[u] = *reinterpret_cast<const float4*>(vb + (size_t)j * HD);
    }
#pragma unroll
    for (int u = 0; u < ATD_UNROLL; ++u) {
      float s = q.x * kv[u].x + q.y * kv[u].y + q.z * kv[u].z + q.w * kv[u].w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (j0 + u < n) {
        s *= scale;
        const float mn = fmaxf(m, s);
        const float corr = expf(m - mn), p = expf(s - mn);
        sum = sum * corr + p;
        o.x = o.x * corr + p * vv[u].x;
        o.y = o.y * corr + p * vv[u].y;
        o.z = o.z * corr + p * vv[u].z;
        o.w = o.w * corr + p * vv[u].w;
        m = mn;
      }
    }
  }
  if (lane == 0) { sm_m[warp] = m; sm_l[warp] = sum; }
  sm_o[warp][lane] = o;
  __syncthreads();
  if (warp == 0) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < ATD_WARPS; ++w) mx = fmaxf(mx, sm_m[w]);
    float tot = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < ATD_WARPS; ++w) {
      const float c = sm_m[w] == -INFINITY ? 0.f : expf(sm_m[w] - mx);
      tot += sm_l[w] * c;
      const float4 ow = sm_o[w][lane];
      acc.x += ow.x * c; acc.y += ow.y * c; acc.z += ow.z * c; acc.w += ow.w * c;
    }
    const float inv = 1.0f / tot;
    *reinterpret_cast<float4*>(A + (size_t)r * HD + h * ATT_D + 4 * lane) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

// ---------------------------------------------------------------------------
// many queries per sequence (prefill): one CTA of 256 threads per (block of QB
// queries, head, sequence), as two key groups of 128 threads: group g takes
// the key blocks g, g + 2, g + 4, ... of KB keys, each with its own double-
// buffered keys and values (16-byte asynchronous copies) and its own running
// softmax; the two partial softmaxes are merged at the end.  Register
// blocking inside a group: thread (q, k) (q < 16, k < 8) computes the scores
// of queries q + 16 r (r < RQ) and keys k + 8 c (c < KC) as outer products of
// float4 reads (broadcast or conflict-free), keeps the running softmax of its
// RQ query rows with the row's 8 lanes (shuffles), and accumulates P V for its
// RQ queries and 16 dimensions 32 i + 4 k .. + 3 (i < 4).
// The tile used: 64 queries (RQ = 4) and key blocks of 32 (KC = 4), ~190
// registers a thread and ~182 KB, one CTA per SM.
// ---------------------------------------------------------------------------
constexpr int ATP_GT = 128;                        // threads per key group
constexpr int ATP_G = 2;                           // key groups per CTA
constexpr int ATP_THREADS = ATP_GT * ATP_G;
constexpr int ATP_PITCH = ATT_D + 4;               // floats per staged row

template <int RQ, int KC>
struct AtpCfg {
  static constexpr int QB = 16 * RQ;               // queries per CTA
  static constexpr int KB = 8 * KC;                // keys per block
  static constexpr int PPITCH = QB + 4;            // probabilities, [key][query]
  static constexpr int GFLOATS = 4 * KB * ATP_PITCH + KB * PPITCH;   // a group's keys, values, probabilities
  static constexpr size_t SMEM = ((size_t)QB * ATP_PITCH + (size_t)ATP_G * GFLOATS) * 4;
  static_assert(ATP_GT * (2 * RQ + 16 * RQ) <= 4 * KB * ATP_PITCH, "a group's softmax state fits its buffers");
};

// 16-byte asynchronous copies of key/value rows j0 .. j0+KB-1 (rows past nk
// zero) by the 128 threads of one key group (gt = thread inside the group).
template <int KB>
BN_DEV void att_stage_kv(const float* kbase, const float* vbase, int HD, int j0, int nk, float* ks, float* vs,
                         int gt) {
  for (int e = gt; e < KB * (ATT_D / 4); e += ATP_GT) {
    const int rr = e / (ATT_D / 4), cc = e - rr * (ATT_D / 4);
    const bool in = rr < nk;
    const size_t off = in ? (size_t)(j0 + rr) * HD + 4 * cc : 0;
    cp_async_16(smem_u32(ks + rr * ATP_PITCH + 4 * cc), kbase + off, in ? 16u : 0u);
    cp_async_16(smem_u32(vs + rr * ATP_PITCH + 4 * cc), vbase + off, in ? 16u : 0u);
  }
  cp_async_commit();
}

// Barrier of one key group's 128 threads (barrier 1 + g; immediate ids, so
// the CTA holds three hardware barriers, not all sixteen).
BN_DEV void att_group_sync(int g) {
  if (g == 0) asm volatile("bar.sync 1, %0;" :: "n"(ATP_GT) : "memory");
  else asm volatile("bar.sync 2, %0;" :: "n"(ATP_GT) : "memory");
}

// Running softmax state of RQ query rows of one thread: max, sum and the
// unnormalised P V of its 16 dimensions.
template <int RQ>
struct AttState {
  float m[RQ], sum[RQ];
  float o[RQ][4][4];                                 // [query r][dimension group i][4]
};

template <int RQ>
BN_DEV void att_state_init(AttState<RQ>& st) {
#pragma unroll
  for (int r = 0; r < RQ; ++r) {
    st.m[r] = -INFINITY;
    st.sum[r] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) st.o[r][i][c] = 0.f;
  }
}

// st <- the merge of st and the state stored at x (field f at x[f * ATP_GT]):
// both rescaled to the larger max (exact in real arithmetic), an empty state
// (max -inf) weighing nothing.
template <int RQ, typename Ld>
BN_DEV void att_state_merge(AttState<RQ>& st, Ld ld) {
#pragma unroll
  for (int r = 0; r < RQ; ++r) {
    const float m1 = ld(2 * r), s1 = ld(2 * r + 1);
    const float mn = fmaxf(st.m[r], m1);
    const float c0 = st.m[r] == -INFINITY ? 0.f : expf(st.m[r] - mn);
    const float c1 = m1 == -INFINITY ? 0.f : expf(m1 - mn);
    st.sum[r] = st.sum[r] * c0 + s1 * c1;
    st.m[r] = mn;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) st.o[r][i][c] = st.o[r][i][c] * c0 + ld(2 * RQ + 16 * r + 4 * i + c) * c1;
  }
}

// Key blocks [kb0, kb1) of query block qb for the whole CTA: the queries are
// staged, group g takes the blocks kb0 + g, kb0 + g + 2, ..., and at the end
// group 1's state is merged into group 0's (st is valid in group 0 only).
// Every thread of the CTA calls it with the same arguments.
template <int RQ, int KC>
BN_DEV void att_task(const float* __restrict__ Q, const float* __restrict__ kbase, const float* __restrict__ vbase,
                     int b, int h, int L, int t0, int HD, float scale, int qb, int kb0, int kb1, float* atp,
                     AttState<RQ>& st) {
  using C = AtpCfg<RQ, KC>;
  constexpr int QB = C::QB, KB = C::KB, PPITCH = C::PPITCH, GFLOATS = C::GFLOATS;
  const int tid = threadIdx.x;
  const int g = tid / ATP_GT, gt = tid - g * ATP_GT;
  const int tq = gt >> 3, tk = gt & 7;
  float* qs = atp;                                  // [QB][PITCH]
  float* kbuf = qs + QB * ATP_PITCH + g * GFLOATS;  // [2][KB][PITCH] of this group
  float* vbuf = kbuf + 2 * KB * ATP_PITCH;          // [2][KB][PITCH]
  float* pt = vbuf + 2 * KB * ATP_PITCH;            // [KB][PPITCH] probabilities of the current block
  const int l0 = qb * QB;
  const int nq = L - l0 < QB ? L - l0 : QB;
  const int kend = t0 + l0 + nq;                     // keys 0 .. kend-1 are visible to the block
  __syncthreads();                                   // the previous task is done with every buffer
  att_state_init(st);
  if (kb0 + g < kb1) {
    const int j0 = (kb0 + g) * KB;
    att_stage_kv<KB>(kbase, vbase, HD, j0, kend - j0 < KB ? kend - j0 : KB, kbuf, vbuf, gt);
  }
  for (int e = tid; e < QB * (ATT_D / 4); e += ATP_THREADS) {
    const int rr = e / (ATT_D / 4), cc = e - rr * (ATT_D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < nq) v = *reinterpret_cast<const float4*>(Q + ((size_t)b * L + l0 + rr) * HD + h * ATT_D + 4 * cc);
    *reinterpret_cast<float4*>(qs + rr * ATP_PITCH + 4 * cc) = v;
  }
  __syncthreads();                                   // the queries are in place for both groups
  for (int blk = kb0 + g, it = 0; blk < kb1; blk += ATP_G, ++it) {
    const int j0 = blk * KB;
    const int nk = kend - j0 < KB ? kend - j0 : KB;
    if (blk + ATP_G < kb1) {
      const int j1 = j0 + ATP_G * KB;
      att_stage_kv<KB>(kbase, vbase, HD, j1, kend - j1 < KB ? kend - j1 : KB,
                       kbuf + ((it + 1) & 1) * KB * ATP_PITCH, vbuf + ((it + 1) & 1) * KB * ATP_PITCH, gt);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      cp_async_wait_all();
    }
    att_group_sync(g);                               // this block's K and V are in place
    const float* ks = kbuf + (it & 1) * KB * ATP_PITCH;
    const float* vs = vbuf + (it & 1) * KB * ATP_PITCH;
    // ---- scores of queries tq + 16 r and keys tk + 8 c ----
    float sc[RQ][KC];
#pragma unroll
    for (int r = 0; r < RQ; ++r)
#pragma unroll
      for (int c = 0; c < KC; ++c) sc[r][c] = 0.f;
#pragma unroll 4
    for (int dd = 0; dd < ATT_D; dd += 4) {
      float4 qv[RQ], kv[KC];
#pragma unroll
      for (int r = 0; r < RQ; ++r) qv[r] = *reinterpret_cast<const float4*>(qs + (tq + 16 * r) * ATP_PITCH + dd);
#pragma unroll
      for (int c = 0; c < KC; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (tk + 8 * c) * ATP_PITCH + dd);
#pragma unroll
      for (int r = 0; r < RQ; ++r)
#pragma unroll
        for (int c = 0; c < KC; ++c)
          sc[r][c] += qv[r].x * kv[c].x + qv[r].y * kv[c].y + qv[r].z * kv[c].z + qv[r].w * kv[c].w;
    }
    // ---- running softmax of the query rows (the row's 8 lanes: xor 1, 2, 4) ----
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
      const int qpos = t0 + l0 + tq + 16 * r;
      float bm = -INFINITY;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const int jj = tk + 8 * c;
        sc[r][c] = (jj < nk && j0 + jj <= qpos) ? sc[r][c] * scale : -INFINITY;
        bm = fmaxf(bm, sc[r][c]);
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      const float mn = fmaxf(st.m[r], bm);
      // a query row whose keys in this block are all masked keeps its state
      const float corr = mn == -INFINITY ? 1.f : expf(st.m[r] - mn);
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const float pp = sc[r][c] == -INFINITY ? 0.f : expf(sc[r][c] - mn);
        pt[(tk + 8 * c) * PPITCH + tq + 16 * r] = pp;
        psum += pp;
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      st.sum[r] = st.sum[r] * corr + psum;
      st.m[r] = mn;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) st.o[r][i][c] *= corr;
    }
    att_group_sync(g);                               // every row's probabilities are in place
    // ---- P V: queries tq + 16 r, dimensions 32 i + 4 tk .. + 3 ----
#pragma unroll 2
    for (int j = 0; j < nk; ++j) {
      float pr[RQ];
#pragma unroll
      for (int r = 0; r < RQ; ++r) pr[r] = pt[j * PPITCH + tq + 16 * r];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(vs + j * ATP_PITCH + 32 * i + 4 * tk);
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
          st.o[r][i][0] += pr[r] * v.x; st.o[r][i][1] += pr[r] * v.y;
          st.o[r][i][2] += pr[r] * v.z; st.o[r][i][3] += pr[r] * v.w;
        }
      }
    }
    att_group_sync(g);                               // every thread of the group is done with this block's buffers
  }
  // ---- group 1 hands its state to the same thread of group 0 ----
  float* xch = atp + QB * ATP_PITCH + GFLOATS;       // group 1's key/value buffers (no copy in flight)
  if (g == 1) {
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
      xch[(2 * r) * ATP_GT + gt] = st.m[r];
      xch[(2 * r + 1) * ATP_GT + gt] = st.sum[r];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) xch[(2 * RQ + 16 * r + 4 * i + c) * ATP_GT + gt] = st.o[r][i][c];
    }
  }
  __syncthreads();
  if (g == 0) att_state_merge<RQ>(st, [&](int f) { return xch[f * ATP_GT + gt]; });
}

// Group 0 writes the normalised output rows of query block qb.
template <int RQ, int KC>
BN_DEV void att_write(const AttState<RQ>& st, float* __restrict__ A, int b, int h, int L, int HD, int qb) {
  using C = AtpCfg<RQ, KC>;
  const int gt = threadIdx.x, tq = gt >> 3, tk = gt & 7;
  const int l0 = qb * C::QB;
  const int nq = L - l0 < C::QB ? L - l0 : C::QB;
#pragma unroll
  for (int r = 0; r < RQ; ++r) {
    const int row = tq + 16 * r;
    const float inv = 1.0f / st.sum[r];
    if (row < nq) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4*>(A + ((size_t)b * L + l0 + row) * HD + h * ATT_D + 4 * tk + 32 * i) =
            make_float4(st.o[r][i][0] * inv, st.o[r][i][1] * inv, st.o[r][i][2] * inv, st.o[r][i][3] * inv);
    }
  }
}

// Causal prefill over clusters of two CTAs per (pair of query blocks, head,
// sequence): query block qa = p (light) and qz = nqb - 1 - p (heavy) have
// nblk(qa) + nblk(qz) key blocks between them, split evenly: CTA 0 takes the
// first s key blocks of qz and then all of qa, CTA 1 the rest of qz.  CTA 0
// stores its partial state of qz into CTA 1's shared memory (distributed
// shared memory), and CTA 1 merges it into its own before writing qz.  (When
// qa == qz, the middle block of an odd count, its keys are split in half.)
template <int RQ, int KC>
__global__ void __launch_bounds__(ATP_THREADS, 1)
attention_prefill_kernel(const float* __restrict__ Q, const float* __restrict__ Kc, const float* __restrict__ Vc,
                         int L, int t0, int HD, int T_cap, float scale, float* __restrict__ A) {
  using C = AtpCfg<RQ, KC>;
  constexpr int QB = C::QB, KB = C::KB;
  extern __shared__ float atp[];
  float* pex = atp + (C::SMEM / 4);                  // [2 RQ + 16 RQ][ATP_GT]: the partner's partial state
  pdl_launch_dependents();
  cluster_arrive();                                  // both CTAs of the pair run before any remote store
  cluster_wait();
  pdl_wait();
  const int rank = blockIdx.x & 1, p = blockIdx.x >> 1, h = blockIdx.y, b = blockIdx.z;
  const int nqb = (L + QB - 1) / QB;
  const int qa = p, qz = nqb - 1 - p;
  auto nblk = [&](int q) {
    const int l0 = q * QB;
    return (t0 + l0 + (L - l0 < QB ? L - l0 : QB) + KB - 1) / KB;
  };
  const int wz = nblk(qz);
  const int s = qa == qz ? wz / 2 : (wz - nblk(qa) > 0 ? (wz - nblk(qa)) / 2 : 0);
  const float* kbase = Kc + (size_t)b * T_cap * HD + h * ATT_D;
  const float* vbase = Vc + (size_t)b * T_cap * HD + h * ATT_D;
  const int gt = threadIdx.x;
  AttState<RQ> st;
  if (rank == 0) {
    att_task<RQ, KC>(Q, kbase, vbase, b, h, L, t0, HD, scale, qz, 0, s, atp, st);
    if (gt < ATP_GT) {                               // group 0 stores its state into the partner's buffer
      const uint32_t dst = cluster_map(smem_u32(pex), 1);
#pragma unroll
      for (int r = 0; r < RQ; ++r) {
        st_cluster_u32(dst + 4u * ((2 * r) * ATP_GT + gt), __float_as_uint(st.m[r]));
        st_cluster_u32(dst + 4u * ((2 * r + 1) * ATP_GT + gt), __float_as_uint(st.sum[r]));
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_cluster_u32(dst + 4u * ((2 * RQ + 16 * r + 4 * i + c) * ATP_GT + gt), __float_as_uint(st.o[r][i][c]));
      }
    }
    cluster_arrive();                                // releases the stores to the partner
    if (qa != qz) {
      att_task<RQ, KC>(Q, kbase, vbase, b, h, L, t0, HD, scale, qa, 0, nblk(qa), atp, st);
      if (gt < ATP_GT) att_write<RQ, KC>(st, A, b, h, L, HD, qa);
    }
    cluster_wait();
  } else {
    att_task<RQ, KC>(Q, kbase, vbase, b, h, L, t0, HD, scale, qz, s, wz, atp, st);
    cluster_arrive();
    cluster_wait();                                  // the partner's state is in place
    if (gt < ATP_GT) {
      att_state_merge<RQ>(st, [&](int f) { return pex[f * ATP_GT + gt]; });
      att_write<RQ, KC>(st, A, b, h, L, HD, qz);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
cudaError_t run_rope_append(float* Q, const float* K, const float* V, int B, int L, int t0, int heads, int d,
                            double base, float* Kc, float* Vc, int T_cap, cudaStream_t st) {
  const int HD = heads * d;
  const size_t total = (size_t)B * L * (HD / 2);
  const unsigned blocks = (unsigned)((total + 255) / 256);
  return launch_pdl(rope_append_kernel, dim3(blocks), dim3(256), 0, st, 1u, Q, K, V, B, L, t0, HD, d, log2(base),
                    Kc, Vc, T_cap);
}

cudaError_t run_attention(const float* Q, const float* Kc, const float* Vc, int B, int L, int t0, int heads, int d,
                          int T_cap, float* A, cudaStream_t st) {
  const int HD = heads * d;
  const float scale = (float)(1.0 / sqrt((double)d));
  if (L < 16) {
    return launch_pdl(attention_decode_kernel, dim3((unsigned)(B * L), (unsigned)heads), dim3(32 * ATD_WARPS), 0, st,
                      1u, Q, Kc, Vc, L, t0, HD, T_cap, scale, A);
  }
  // 64 queries and 32-key blocks.  Measured on B200 (24 layers of a causal
  // 512-token sequence, 16 heads): 2.18 ms; 32 queries and 16-key blocks, at
  // two CTAs per SM and half the heaviest block's serial work, 2.71 ms (twice
  // the shared-memory reads per multiply-add, twice the blocks and barriers).
  using C = AtpCfg<4, 4>;
  auto kern = attention_prefill_kernel<4, 4>;
  const size_t smem = C::SMEM + (size_t)ATP_GT * 18 * 4 * sizeof(float);   // + the partner's partial state
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int nqb = (L + C::QB - 1) / C::QB;
  const int pairs = (nqb + 1) / 2;
  return launch_pdl(kern, dim3((unsigned)(2 * pairs), (unsigned)heads, (unsigned)B), dim3(ATP_THREADS), smem, st,
                    dim3(2, 1, 1), Q, Kc, Vc, L, t0, HD, T_cap, scale, A);
}

}  // namespace bitnet
