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

template <int RQ, int KC>
__global__ void __launch_bounds__(ATP_THREADS, RQ <= 2 ? 2 : 1)
attention_prefill_kernel(const float* __restrict__ Q, const float* __restrict__ Kc, const float* __restrict__ Vc,
                         int L, int t0, int HD, int T_cap, float scale, float* __restrict__ A) {
  using C = AtpCfg<RQ, KC>;
  constexpr int QB = C::QB, KB = C::KB, PPITCH = C::PPITCH, GFLOATS = C::GFLOATS;
  extern __shared__ float atp[];
  const int tid = threadIdx.x;
  const int g = tid / ATP_GT, gt = tid - g * ATP_GT;
  float* qs = atp;                                  // [QB][PITCH]
  float* kbuf = qs + QB * ATP_PITCH + g * GFLOATS;  // [2][KB][PITCH] of this group
  float* vbuf = kbuf + 2 * KB * ATP_PITCH;          // [2][KB][PITCH]
  float* pt = vbuf + 2 * KB * ATP_PITCH;            // [KB][PPITCH] probabilities of the current block
  pdl_launch_dependents();
  pdl_wait();
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int l0 = qb * QB;
  const int nq = L - l0 < QB ? L - l0 : QB;
  const int tq = gt >> 3, tk = gt & 7;
  const float* kbase = Kc + (size_t)b * T_cap * HD + h * ATT_D;
  const float* vbase = Vc + (size_t)b * T_cap * HD + h * ATT_D;
  const int kend = t0 + l0 + nq;                     // keys 0 .. kend-1 are needed by the block
  const int nblk = (kend + KB - 1) / KB;
  if (g < nblk) {
    const int j0 = g * KB;
    att_stage_kv<KB>(kbase, vbase, HD, j0, kend - j0 < KB ? kend - j0 : KB, kbuf, vbuf, gt);
  }
  for (int e = tid; e < QB * (ATT_D / 4); e += ATP_THREADS) {
    const int rr = e / (ATT_D / 4), cc = e - rr * (ATT_D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < nq) v = *reinterpret_cast<const float4*>(Q + ((size_t)b * L + l0 + rr) * HD + h * ATT_D + 4 * cc);
    *reinterpret_cast<float4*>(qs + rr * ATP_PITCH + 4 * cc) = v;
  }
  __syncthreads();                                   // the queries are in place for both groups
  float m[RQ], sum[RQ];
  float o[RQ][4][4];                                 // [query r][dimension group i][4]
#pragma unroll
  for (int r = 0; r < RQ; ++r) {
    m[r] = -INFINITY;
    sum[r] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) o[r][i][c] = 0.f;
  }
  for (int blk = g, it = 0; blk < nblk; blk += ATP_G, ++it) {
    const int j0 = blk * KB;
    const int nk = kend - j0 < KB ? kend - j0 : KB;
    if (blk + ATP_G < nblk) {
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
    float s[RQ][KC];
#pragma unroll
    for (int r = 0; r < RQ; ++r)
#pragma unroll
      for (int c = 0; c < KC; ++c) s[r][c] = 0.f;
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
          s[r][c] += qv[r].x * kv[c].x + qv[r].y * kv[c].y + qv[r].z * kv[c].z + qv[r].w * kv[c].w;
    }
    // ---- running softmax of the query rows (the row's 8 lanes: xor 1, 2, 4) ----
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
      const int qpos = t0 + l0 + tq + 16 * r;
      float bm = -INFINITY;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const int jj = tk + 8 * c;
        s[r][c] = (jj < nk && j0 + jj <= qpos) ? s[r][c] * scale : -INFINITY;
        bm = fmaxf(bm, s[r][c]);
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      const float mn = fmaxf(m[r], bm);
      // a query row whose keys in this block are all masked keeps its state
      const float corr = mn == -INFINITY ? 1.f : expf(m[r] - mn);
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const float p = s[r][c] == -INFINITY ? 0.f : expf(s[r][c] - mn);
        pt[(tk + 8 * c) * PPITCH + tq + 16 * r] = p;
        psum += p;
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      sum[r] = sum[r] * corr + psum;
      m[r] = mn;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[r][i][c] *= corr;
    }
    att_group_sync(g);                               // every row's probabilities are in place
    // ---- P V: queries tq + 16 r, dimensions 32 i + 4 tk .. + 3 ----
#pragma unroll 2
    for (int j = 0; j < nk; ++j) {
      float p[RQ];
#pragma unroll
      for (int r = 0; r < RQ; ++r) p[r] = pt[j * PPITCH + tq + 16 * r];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(vs + j * ATP_PITCH + 32 * i + 4 * tk);
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
          o[r][i][0] += p[r] * v.x; o[r][i][1] += p[r] * v.y; o[r][i][2] += p[r] * v.z; o[r][i][3] += p[r] * v.w;
        }
      }
    }
    att_group_sync(g);                               // every thread of the group is done with this block's buffers
  }
  // ---- merge: group 1 hands its running max, sum and output to the same thread of group 0 ----
  float* xch = atp + QB * ATP_PITCH + GFLOATS;       // group 1's key/value buffers (no copy in flight)
  if (g == 1) {
#pragma unroll
    for (int r = 0; r < RQ; ++r) {
      xch[(2 * r) * ATP_GT + gt] = m[r];
      xch[(2 * r + 1) * ATP_GT + gt] = sum[r];
    }
#pragma unroll
    for (int r = 0; r < RQ; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) xch[(2 * RQ + 16 * r + 4 * i + c) * ATP_GT + gt] = o[r][i][c];
  }
  __syncthreads();
  if (g == 1) return;
#pragma unroll
  for (int r = 0; r < RQ; ++r) {
    const float m1 = xch[(2 * r) * ATP_GT + gt], s1 = xch[(2 * r + 1) * ATP_GT + gt];
    const float mn = fmaxf(m[r], m1);
    const float c0 = m[r] == -INFINITY ? 0.f : expf(m[r] - mn);
    const float c1 = m1 == -INFINITY ? 0.f : expf(m1 - mn);
    const float tot = sum[r] * c0 + s1 * c1;
    const int row = tq + 16 * r;
    const float inv = 1.0f / tot;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* x1 = xch + (2 * RQ + 16 * r + 4 * i) * ATP_GT + gt;
      float4 res;
      res.x = (o[r][i][0] * c0 + x1[0 * ATP_GT] * c1) * inv;
      res.y = (o[r][i][1] * c0 + x1[1 * ATP_GT] * c1) * inv;
      res.z = (o[r][i][2] * c0 + x1[2 * ATP_GT] * c1) * inv;
      res.w = (o[r][i][3] * c0 + x1[3 * ATP_GT] * c1) * inv;
      if (row < nq)
        *reinterpret_cast<float4*>(A + ((size_t)b * L + l0 + row) * HD + h * ATT_D + 4 * tk + 32 * i) = res;
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
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)((L + C::QB - 1) / C::QB), (unsigned)heads, (unsigned)B),
                    dim3(ATP_THREADS), C::SMEM, st, 1u, Q, Kc, Vc, L, t0, HD, T_cap, scale, A);
}

}  // namespace bitnet
