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
// many queries per sequence (prefill): one CTA per (block of 16 queries, head,
// sequence).  Key blocks of 64 keys (and their values) are staged in shared
// memory; 256 threads compute the 16 x 64 scores (4 each), update the running
// softmax of their query row, then accumulate P V (8 output dimensions each).
// ---------------------------------------------------------------------------
constexpr int ATP_QB = 16;
constexpr int ATP_KB = 64;
constexpr int ATP_PITCH = ATT_D + 4;               // floats per staged row (conflict-free float4 reads)
constexpr size_t ATP_SMEM = (size_t)(ATP_QB + 2 * ATP_KB) * ATP_PITCH * 4 + (size_t)ATP_QB * ATP_KB * 4;

__global__ void __launch_bounds__(256, 2)
attention_prefill_kernel(const float* __restrict__ Q, const float* __restrict__ Kc, const float* __restrict__ Vc,
                         int L, int t0, int HD, int T_cap, float scale, float* __restrict__ A) {
  extern __shared__ float atp[];
  float* qs = atp;                                  // [16][PITCH]
  float* ks = qs + ATP_QB * ATP_PITCH;              // [64][PITCH]
  float* vs = ks + ATP_KB * ATP_PITCH;              // [64][PITCH]
  float* ps = vs + ATP_KB * ATP_PITCH;              // [16][64] probabilities of the current block
  pdl_launch_dependents();
  pdl_wait();
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int l0 = qb * ATP_QB;
  const int nq = L - l0 < ATP_QB ? L - l0 : ATP_QB;
  const int tid = threadIdx.x;
  const int row = tid >> 4, c16 = tid & 15;         // query row; column slot
  // queries
  for (int e = tid; e < ATP_QB * (ATT_D / 4); e += 256) {
    const int rr = e / (ATT_D / 4), cc = e - rr * (ATT_D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < nq) v = *reinterpret_cast<const float4*>(Q + ((size_t)b * L + l0 + rr) * HD + h * ATT_D + 4 * cc);
    *reinterpret_cast<float4*>(qs + rr * ATP_PITCH + 4 * cc) = v;
  }
  const int qpos = t0 + l0 + row;                    // this thread's query position
  const int kend = t0 + l0 + nq;                     // keys 0 .. kend-1 are needed by the block
  float m = -INFINITY, sum = 0.f;
  float o[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) o[t] = 0.f;
  const float* kbase = Kc + (size_t)b * T_cap * HD + h * ATT_D;
  const float* vbase = Vc + (size_t)b * T_cap * HD + h * ATT_D;
  for (int j0 = 0; j0 < kend; j0 += ATP_KB) {
    const int nk = kend - j0 < ATP_KB ? kend - j0 : ATP_KB;
    __syncthreads();                                 // the previous block's K, V, P are consumed
    for (int e = tid; e < ATP_KB * (ATT_D / 4); e += 256) {
      const int rr = e / (ATT_D / 4), cc = e - rr * (ATT_D / 4);
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (rr < nk) {
        kv = *reinterpret_cast<const float4*>(kbase + (size_t)(j0 + rr) * HD + 4 * cc);
        vv = *reinterpret_cast<const float4*>(vbase + (size_t)(j0 + rr) * HD + 4 * cc);
      }
      *reinterpret_cast<float4*>(ks + rr * ATP_PITCH + 4 * cc) = kv;
      *reinterpret_cast<float4*>(vs + rr * ATP_PITCH + 4 * cc) = vv;
    }
    __syncthreads();
    // scores of keys c16 + 16 u for this thread's query row
    float s[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) s[u] = 0.f;
    const float* qr = qs + row * ATP_PITCH;
#pragma unroll 8
    for (int dd = 0; dd < ATT_D; dd += 4) {
      const float4 qv = *reinterpret_cast<const float4*>(qr + dd);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 kv = *reinterpret_cast<const float4*>(ks + (c16 + 16 * u) * ATP_PITCH + dd);
        s[u] += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
      }
    }
    float bm = -INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + c16 + 16 * u;
      s[u] = (c16 + 16 * u < nk && j <= qpos) ? s[u] * scale : -INFINITY;
      bm = fmaxf(bm, s[u]);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
    const float mn = fmaxf(m, bm);
    // a query row whose keys in this block are all masked keeps its state
    const float corr = mn == -INFINITY ? 1.f : expf(m - mn);
    float ps_sum = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float p = s[u] == -INFINITY ? 0.f : expf(s[u] - mn);
      ps[row * ATP_KB + c16 + 16 * u] = p;
      ps_sum += p;
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ps_sum += __shfl_xor_sync(0xffffffffu, ps_sum, off);
    sum = sum * corr + ps_sum;
    m = mn;
#pragma unroll
    for (int t = 0; t < 8; ++t) o[t] *= corr;
    __syncwarp();
    // P V for dimensions 8 c16 .. 8 c16 + 7 of this query row
    const float* pr = ps + row * ATP_KB;
    for (int j = 0; j < nk; ++j) {
      const float p = pr[j];
      const float4 v0 = *reinterpret_cast<const float4*>(vs + j * ATP_PITCH + 8 * c16);
      const float4 v1 = *reinterpret_cast<const float4*>(vs + j * ATP_PITCH + 8 * c16 + 4);
      o[0] += p * v0.x; o[1] += p * v0.y; o[2] += p * v0.z; o[3] += p * v0.w;
      o[4] += p * v1.x; o[5] += p * v1.y; o[6] += p * v1.z; o[7] += p * v1.w;
    }
  }
  if (row < nq) {
    const float inv = 1.0f / sum;
    float* dst = A + ((size_t)b * L + l0 + row) * HD + h * ATT_D + 8 * c16;
    *reinterpret_cast<float4*>(dst) = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(o[4] * inv, o[5] * inv, o[6] * inv, o[7] * inv);
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
  if (L < ATP_QB) {
    return launch_pdl(attention_decode_kernel, dim3((unsigned)(B * L), (unsigned)heads), dim3(32 * ATD_WARPS), 0, st,
                      1u, Q, Kc, Vc, L, t0, HD, T_cap, scale, A);
  }
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(attention_prefill_kernel), ATP_SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(attention_prefill_kernel, dim3((unsigned)((L + ATP_QB - 1) / ATP_QB), (unsigned)heads, (unsigned)B),
                    dim3(256), ATP_SMEM, st, 1u, Q, Kc, Vc, L, t0, HD, T_cap, scale, A);
}

}  // namespace bitnet
