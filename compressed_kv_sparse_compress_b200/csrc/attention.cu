// Step 3 of the decode path: joint attention over the selected compressed entries and the
// sliding window, with one shared K=V vector per key and inverse RoPE on the output.
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": shared K=V vectors with inverse RoPE, sparse attention over the
// top-k compressed tokens, a local window of full vectors. Reading: one softmax over the union
// of the selected entries and the window tokens [max(0, L-W), L), without de-duplication.
//
// The key list of request b is: selected entries (or all floor(L/r) for a dense layer), then the
// window tokens. It is cut into splits of keys_per_split keys; each split writes an
// un-normalised partial (running max m, sum l, sum of p*x) per head, and attn_combine merges
// the splits by log-sum-exp, normalises, and rotates the rotary dims back by -(L-1).
//
// This file holds the query preparation, the CUDA-core path (any head count, fp32 accumulation of
// everything, fp32 partials) and the two combines. The tensor-core path for H=64, D=512 lives in
// attention_tc.cu and writes the same partials as fp16 rows with a power-of-two scale each.

#include "ckv_internal.h"
#include "query_prep.cuh"
#include "qimage.cuh"
#include "ckv_ptx.cuh"

namespace ckv {

int attention_tc_keys_per_split(int batch, int64_t max_keys);
cudaError_t launch_attention_tc(const LayerParams& p, int batch, const int32_t* seq_len,
                                int max_seq_len, const float* q, const int32_t* idx,
                                const int32_t* cnt, int idx_stride, const AttnWs& ws,
                                uint32_t* status, cudaStream_t stream, bool early, bool rope_ready);

namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtKeys = 32;  // keys per split of the CUDA-core path

struct KeyList {
  int64_t n_c, n_sel, n_win, n_keys;
};

__device__ __forceinline__ KeyList key_list(const LayerParams& p, int L, const int32_t* cnt,
                                            bool sparse, int idx_stride, int b) {
  KeyList k;
  k.n_c = L / p.r;
  k.n_sel = sparse ? min(static_cast<int64_t>(max(cnt[b], 0)), static_cast<int64_t>(idx_stride)) : k.n_c;
  k.n_win = min(p.W, L);
  k.n_keys = k.n_sel + k.n_win;
  return k;
}

// Decodes pair pr (dims 2pr, 2pr+1) of compressed row `row`.
__device__ __forceinline__ float2 comp_pair(const LayerParams& p, int64_t row, int pr) {
  const uint8_t* base = p.comp_codes + row * p.comp_row_bytes;
  if (p.comp_dtype == CKV_F32) return reinterpret_cast<const float2*>(base)[pr];
  if (p.comp_dtype == CKV_BF16) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(base)[pr];
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  const float s = e4m3_to_f32(p.comp_scales[row * (p.D / 16) + pr / 8]);
  const float2 v = __half22float2(e2m1x2_to_half2(base[pr]));
  return make_float2(v.x * s, v.y * s);
}

__device__ __forceinline__ float2 win_pair(const LayerParams& p, int64_t row, int pr) {
  const uint8_t* base = p.win_codes + row * p.win_row_bytes;
  if (p.win_dtype == CKV_F32) return reinterpret_cast<const float2*>(base)[pr];
  const uint16_t c = reinterpret_cast<const uint16_t*>(base)[pr];
  const float s = p.win_scales[row];
  return make_float2(e4m3_to_f32(c & 0xff) * s, e4m3_to_f32(c >> 8) * s);
}

template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const float* q, const int32_t* idx,
    const int32_t* cnt, int idx_stride, AttnWs ws, uint32_t* status) {
  griddep_wait();
  griddep_launch();
  constexpr int NPL = D / 64;  // rotary-aligned pairs per lane
  extern __shared__ float xs[];  // [kSimtKeys][D]
  __shared__ int valid[kSimtKeys];
  const int b = blockIdx.y, s = blockIdx.x;
  const int L = seq_len[b];
  if (L < 1 || L > max_seq_len) return;  // flagged by the combine
  const KeyList kl = key_list(p, L, cnt, idx != nullptr, idx_stride, b);
  const int64_t k0 = static_cast<int64_t>(s) * kSimtKeys;
  if (k0 >= kl.n_keys) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // key i = thread / 8, resolved by its 8 threads together (the same index and table words) and
  // loaded by them a pair of dims at a time: every key's dependent loads are in flight at once
  {
    static_assert(kSimtThreads == 8 * kSimtKeys, "8 threads per key");
    const int i = threadIdx.x >> 3, r = threadIdx.x & 7;
    const int64_t kk = k0 + i;
    bool ok = kk < kl.n_keys;
    int64_t row = -1;
    bool is_win = false;
    if (ok && kk < kl.n_sel) {
      const int64_t ent = idx ? idx[static_cast<int64_t>(b) * idx_stride + kk] : kk;
      if (ent < 0 || ent >= kl.n_c) {
        if (r == 0) atomicOr(status, CKV_DEV_BAD_INDEX);
        ok = false;
      } else {
        row = comp_row(p, b, ent, status);
      }
    } else if (ok) {
      is_win = true;
      row = win_row(p, b, L - kl.n_win + (kk - kl.n_sel), status);
    }
    ok = ok && row >= 0;
    if (ok) {
      for (int pr = r; pr < D / 2; pr += 8)
        reinterpret_cast<float2*>(xs + i * D)[pr] = is_win ? win_pair(p, row, pr) : comp_pair(p, row, pr);
    }
    if (r == 0) valid[i] = ok;
  }
  __syncthreads();

  // the query rotated with the cos/sin table of the rotary pairs, which the query pass (or the prep
  // kernel) wrote before this kernel
  const int first_rope = (D - p.d_r) / 2;
  const double* rope = ws.rope + static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2;
  for (int h = warp; h < p.H; h += kSimtThreads / 32) {
    const float* qh = q + (static_cast<int64_t>(b) * p.H + h) * D;
    float2 qv[NPL], ov[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int pr = lane + 32 * k;
      float2 v = reinterpret_cast<const float2*>(qh)[pr];
      if (pr >= first_rope) {
        const double cs = rope[2 * (pr - first_rope)], sn = rope[2 * (pr - first_rope) + 1];
        const double a0 = v.x, a1 = v.y;
        v = make_float2(static_cast<float>(a0 * cs - a1 * sn), static_cast<float>(a0 * sn + a1 * cs));
      }
      qv[k] = v;
      ov[k] = make_float2(0.f, 0.f);
    }
    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < kSimtKeys; ++i) {
      if (!valid[i]) continue;
      const float2* x = reinterpret_cast<const float2*>(xs + i * D);
      float dot = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const float2 xv = x[lane + 32 * k];
        dot = fmaf(qv[k].x, xv.x, dot);
        dot = fmaf(qv[k].y, xv.y, dot);
      }
      dot = warp_sum(dot) * p.sm_scale;
      const float m_new = fmaxf(m, dot);
      const float alpha = expf(m - m_new);
      const float pj = expf(dot - m_new);
      l = l * alpha + pj;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const float2 xv = x[lane + 32 * k];
        ov[k].x = fmaf(pj, xv.x, ov[k].x * alpha);
        ov[k].y = fmaf(pj, xv.y, ov[k].y * alpha);
      }
      m = m_new;
    }
    const int64_t slot = (static_cast<int64_t>(b) * ws.splits + s) * p.H + h;
#pragma unroll
    for (int k = 0; k < NPL; ++k) reinterpret_cast<float2*>(ws.part_o + slot * D)[lane + 32 * k] = ov[k];
    if (lane == 0) reinterpret_cast<float2*>(ws.part_ml)[slot] = make_float2(m, l);
  }
}

// Query preparation of one part of one request: prep_part (query_prep.cuh).
__global__ void __launch_bounds__(kPrepThreads) attn_prep_kernel(LayerParams p, const int32_t* seq_len,
                                                                 int max_seq_len, const float* q,
                                                                 AttnWs ws) {
  griddep_wait();
  griddep_launch();
  prep_part(p, seq_len, max_seq_len, ws, blockIdx.x, blockIdx.y, threadIdx.x);
}

// Merge of the splits of one (request, head) and inverse rotation for the CUDA-core path (fp32
// partials), one thread per rotary-aligned pair of dims (D/2 threads). Every thread issues the
// loads of its pair's partials for the first kCombineBatch splits before the split weights are
// known; meanwhile the block reduces the splits' (m, l): M = max_s m_s, w_s = exp(m_s - M),
// Z = sum_s w_s l_s (log-sum-exp merge).
constexpr int kCombineBatch = 8;
constexpr int kCombineSmemSplits = 1024;

__global__ void __launch_bounds__(512, 3) attn_combine_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const int32_t* cnt, bool sparse,
    int idx_stride, AttnWs ws, float* out, uint32_t* status) {
  griddep_wait();
  griddep_launch();
  __shared__ float wts[kCombineSmemSplits];
  __shared__ float red[2][16];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int D = p.D, pr = tid;  // dims 2pr, 2pr + 1
  float2* o = reinterpret_cast<float2*>(out + (static_cast<int64_t>(b) * p.H + h) * D);
  const int L = seq_len[b];
  if (L < 1 || L > max_seq_len) {
    if (h == 0 && tid == 0) atomicOr(status, CKV_DEV_BAD_LENGTH);
    o[pr] = make_float2(0.f, 0.f);
    return;
  }
  const int first_rope = (D - p.d_r) / 2;
  double rc = 1.0, rs = 0.0;  // rotation of this pair by the query position
  if (pr >= first_rope) {
    const double* rope = ws.rope + static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2;
    rc = rope[2 * (pr - first_rope)];
    rs = rope[2 * (pr - first_rope) + 1];
  }
  const KeyList kl = key_list(p, L, cnt, sparse, idx_stride, b);
  const int ns = static_cast<int>((kl.n_keys + ws.keys_per_split - 1) / ws.keys_per_split);
  const int64_t base = static_cast<int64_t>(b) * ws.splits;
  const int64_t split_stride = static_cast<int64_t>(p.H) * D / 2;  // in pairs
  const float2* po = reinterpret_cast<const float2*>(ws.part_o + (base * p.H + h) * D) + pr;
  // this pair's partials of the first splits: in flight while the weights are reduced
  float2 x[kCombineBatch];
#pragma unroll
  for (int u = 0; u < kCombineBatch; ++u) x[u] = u < ns ? __ldcg(po + u * split_stride) : make_float2(0.f, 0.f);

  const float2* ml = reinterpret_cast<const float2*>(ws.part_ml);
  float mloc = -INFINITY;
  for (int sidx = tid; sidx < ns; sidx += blockDim.x) {
    const float2 v = __ldcg(ml + (base + sidx) * p.H + h);
    if (v.y > 0.f) mloc = fmaxf(mloc, v.x);  // l = 0: the split holds no keys (or gave up)
  }
  mloc = warp_max(mloc);
  if (lane == 0) red[0][warp] = mloc;
  __syncthreads();
  float M = -INFINITY;
  for (int i = 0; i < nw; ++i) M = fmaxf(M, red[0][i]);
  float zloc = 0.f;
  for (int sidx = tid; sidx < ns; sidx += blockDim.x) {
    const float2 v = __ldcg(ml + (base + sidx) * p.H + h);
    float wv = 0.f;
    if (v.y > 0.f) {
      wv = expf(v.x - M);
      zloc = fmaf(wv, v.y, zloc);
    }
    if (sidx < kCombineSmemSplits) wts[sidx] = wv;
  }
  zloc = warp_sum(zloc);
  if (lane == 0) red[1][warp] = zloc;
  __syncthreads();
  float Z = 0.f;
  for (int i = 0; i < nw; ++i) Z += red[1][i];
  auto weight = [&](int sidx) -> float {
    if (sidx < kCombineSmemSplits) return wts[sidx];
    const float2 v = __ldcg(ml + (base + sidx) * p.H + h);
    if (!(v.y > 0.f)) return 0.f;
    return expf(v.x - M);
  };
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kCombineBatch; ++u) {
    if (u < ns) {
      const float wv = weight(u);
      if (wv > 0.f) {
        acc.x = fmaf(wv, x[u].x, acc.x);
        acc.y = fmaf(wv, x[u].y, acc.y);
      }
    }
  }
  for (int s0 = kCombineBatch; s0 < ns; s0 += kCombineBatch) {
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u)
      x[u] = s0 + u < ns ? __ldcg(po + (s0 + u) * split_stride) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      if (s0 + u < ns) {
        const float wv = weight(s0 + u);
        if (wv > 0.f) {
          acc.x = fmaf(wv, x[u].x, acc.x);
          acc.y = fmaf(wv, x[u].y, acc.y);
        }
      }
    }
  }
  const float inv = Z > 0.f ? 1.f / Z : 0.f;
  float vx = acc.x * inv, vy = acc.y * inv;
  if (pr >= first_rope) {  // inverse rotation
    const double a0 = vx, e0 = vy;
    vx = static_cast<float>(a0 * rc + e0 * rs);
    vy = static_cast<float>(e0 * rc - a0 * rs);
  }
  o[pr] = make_float2(vx, vy);
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t u) {
  __half2_raw hr;
  hr.x = static_cast<unsigned short>(u & 0xffffu);
  hr.y = static_cast<unsigned short>(u >> 16);
  return __half22float2(__half2(hr));
}

// Merge for the tensor-core path (H = 64, D = 512): split s of request b holds O_s as fp16 rows of 64
// heads per dim (part_h[b][s][d][h], head h divided by part_sc[b][s][h]) and (m, l) per head with
// the maximum in base 2. One CTA per (request, block of 16 dims); thread t merges heads
// 2 (t % 32), 2 (t % 32) + 1 over dims 4 ((t / 32) % 4) .. + 3 of the block (a warp reads 128
// contiguous bytes per dim) for the splits of its group g = t / 128 (splits g, g + G, g + 2 G, ..):
// each of the G split groups keeps its own running maximum, sum and accumulators, reading the
// partials from L2 kBatch splits at a time, and group 0 merges them in shared memory (log-sum-exp).
// G = 4 when the requests have more than 16 splits, else 1.
//
// The length, the selection count and (rope_ready: written by a kernel before the attention) the
// cos/sin table are read before the wait: this kernel starts only once every attention CTA that
// holds keys has passed its own wait, which in turn follows the kernels that wrote them.
constexpr int kGDim = 512;
constexpr int kGHeads = 64;
constexpr int kGDimsPerCta = 16;
constexpr int kGBatch = 8;       // splits whose loads are in flight together (one group)
constexpr int kGBatchMany = 9;   // the same, per group of four

template <int kGGroups, int kBatch>
__global__ void __launch_bounds__(128 * kGGroups) attn_combine_tc_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const int32_t* cnt, bool sparse,
    int idx_stride, AttnWs ws, float* out, uint32_t* status, bool rope_ready) {
  __shared__ float4 red_acc[kGGroups > 1 ? kGGroups - 1 : 1][128][2];  // groups 1..: the two heads' accumulators
  __shared__ float4 red_mz[kGGroups > 1 ? kGGroups - 1 : 1][128];      // (M0, Z0, M1, Z1)
  const int blk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int hp = tid & 31, sg = tid >> 7, tg = tid & 127;
  const int d0 = kGDimsPerCta * blk + 4 * ((tid >> 5) & 3);
  const int L = __ldcg(seq_len + b);
  const bool live = L >= 1 && L <= max_seq_len;
  const int sel = live && sparse ? __ldcg(cnt + b) : 0;
  // cos, sin of the rotary pairs d0 / 2, d0 / 2 + 1 (inverse rotation of group 0's outputs)
  const int first_rope = (kGDim - p.d_r) / 2;
  const double* rope = ws.rope + static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2;
  double cs[2] = {1.0, 1.0}, sn[2] = {0.0, 0.0};
  auto load_rope = [&]() {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int pr = d0 / 2 + k;
      if (pr >= first_rope) {
        cs[k] = __ldcg(rope + 2 * (pr - first_rope));
        sn[k] = __ldcg(rope + 2 * (pr - first_rope) + 1);
      }
    }
  };
  if (rope_ready && live && sg == 0) load_rope();
  griddep_wait();
  griddep_launch();
  float4* o0 = reinterpret_cast<float4*>(out + (static_cast<int64_t>(b) * kGHeads + 2 * hp) * kGDim + d0);
  float4* o1 = o0 + kGDim / 4;
  if (!live) {
    if (blk == 0 && tid == 0) atomicOr(status, CKV_DEV_BAD_LENGTH);
    if (sg == 0) *o0 = *o1 = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  if (!rope_ready && sg == 0) load_rope();
  const int64_t n_c = L / p.r;
  const int64_t n_keys = (sparse ? min(static_cast<int64_t>(max(sel, 0)), static_cast<int64_t>(idx_stride)) : n_c) +
                         min(p.W, L);
  const int ns = static_cast<int>((n_keys + ws.keys_per_split - 1) / ws.keys_per_split);
  const int64_t base = static_cast<int64_t>(b) * ws.splits;
  const float4* ml = reinterpret_cast<const float4*>(ws.part_ml);           // (m, l) of 2 heads
  const float2* scp = reinterpret_cast<const float2*>(ws.part_sc);          // scales of 2 heads
  const uint32_t* ph = reinterpret_cast<const uint32_t*>(ws.part_h);        // fp16 pairs of heads
  float M[2] = {-INFINITY, -INFINITY}, Z[2] = {0.f, 0.f}, acc[2][4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[0][k] = acc[1][k] = 0.f;
  // merge (m, l, x) of one split into this thread's running state (j: head of the pair)
  auto merge = [&](int j, float m, float l, float w_scale, const float (&x)[4]) {
    if (!(l > 0.f)) return;  // l = 0: the split holds no keys (or gave up)
    if (m > M[j]) {          // a new maximum: rescale what is merged so far
      const float f = M[j] == -INFINITY ? 0.f : exp2f(M[j] - m);
      Z[j] *= f;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[j][k] *= f;
      M[j] = m;
    }
    const float w = exp2f(m - M[j]);
    Z[j] = fmaf(w, l, Z[j]);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[j][k] = fmaf(w * w_scale, x[k], acc[j][k]);
  };
  for (int i0 = 0; sg + kGGroups * i0 < ns; i0 += kBatch) {
    float4 v[kBatch];
    float2 sc[kBatch];
    uint32_t x[kBatch][4];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int s = sg + kGGroups * (i0 + u);
      if (s < ns) {
        const int64_t slot = base + s;
        v[u] = __ldcg(ml + slot * (kGHeads / 2) + hp);
        sc[u] = __ldcg(scp + slot * (kGHeads / 2) + hp);
#pragma unroll
        for (int k = 0; k < 4; ++k) x[u][k] = __ldcg(ph + (slot * kGDim + d0 + k) * (kGHeads / 2) + hp);
      } else {
        v[u] = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      float xa[4], xb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 xf = half2_bits_to_float2(x[u][k]);
        xa[k] = xf.x;
        xb[k] = xf.y;
      }
      merge(0, v[u].x, v[u].y, sc[u].x, xa);
      merge(1, v[u].z, v[u].w, sc[u].y, xb);
    }
  }
  // groups 1.. hand their state to group 0
  if (kGGroups > 1 && sg > 0) {
    red_mz[sg - 1][tg] = make_float4(M[0], Z[0], M[1], Z[1]);
    red_acc[sg - 1][tg][0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
    red_acc[sg - 1][tg][1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
  }
  if (kGGroups > 1) {
    __syncthreads();
    if (sg > 0) return;
  }
#pragma unroll
  for (int g = 0; g < kGGroups - 1; ++g) {
    const float4 mz = red_mz[g][tg];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float m = j ? mz.z : mz.x, z = j ? mz.w : mz.y;
      if (!(z > 0.f)) continue;
      const float4 a = red_acc[g][tg][j];
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float Mn = fmaxf(M[j], m);
      const float f_self = M[j] == -INFINITY ? 0.f : exp2f(M[j] - Mn), f_other = exp2f(m - Mn);
      Z[j] = Z[j] * f_self + z * f_other;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[j][k] = acc[j][k] * f_self + av[k] * f_other;
      M[j] = Mn;
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float4* o = j ? o1 : o0;
    if (!(Z[j] > 0.f)) {  // no key: a zero output
      *o = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const float inv = 1.f / Z[j];
    float v4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v4[k] = acc[j][k] * inv;
#pragma unroll
    for (int k = 0; k < 2; ++k) {  // inverse rotation by the query position
      if (d0 / 2 + k >= first_rope) {
        const double a0 = v4[2 * k], e0 = v4[2 * k + 1];
        v4[2 * k] = static_cast<float>(a0 * cs[k] + e0 * sn[k]);
        v4[2 * k + 1] = static_cast<float>(e0 * cs[k] - a0 * sn[k]);
      }
    }
    *o = make_float4(v4[0], v4[1], v4[2], v4[3]);
  }
}

template <int D>
cudaError_t launch_simt_d(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                          const float* q, const int32_t* idx, const int32_t* cnt, int idx_stride,
                          const AttnWs& ws, uint32_t* status, cudaStream_t stream) {
  const int smem = kSimtKeys * D * static_cast<int>(sizeof(float));
  auto kern = attn_simt_kernel<D>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ws.splits, batch);
  return launch_kernel(kern, grid, dim3(kSimtThreads), smem, stream, p, seq_len, max_seq_len, q, idx,
                       cnt, idx_stride, ws, status);
}

}  // namespace

AttnWs attention_ws_layout(void* base, const LayerParams& p, int batch, int max_seq_len,
                           int max_selected) {
  AttnWs w{};
  const int64_t sel = max_selected > 0 ? max_selected : static_cast<int64_t>(max_seq_len) / p.r;
  const int64_t keys = sel + (p.W < max_seq_len ? p.W : max_seq_len);
  w.keys_per_split = attention_tc_supported(p)
                         ? attention_tc_keys_per_split(batch, keys)
                         : kSimtKeys;
  w.splits = static_cast<int>(keys > 0 ? (keys + w.keys_per_split - 1) / w.keys_per_split : 1);
  const size_t n_slot = static_cast<size_t>(batch) * w.splits * p.H;
  const size_t o_bytes = align_up(n_slot * p.D * sizeof(float), 256);
  const size_t ml_bytes = align_up(n_slot * 2 * sizeof(float), 256);
  const size_t sc_bytes = align_up(n_slot * sizeof(float), 256);
  const size_t rope_bytes = align_up(static_cast<size_t>(batch) * (p.d_r / 2 + 1) * 2 * sizeof(double), 256);
  w.half_parts = attention_tc_supported(p);
  const size_t qi_bytes = w.half_parts ? align_up(static_cast<size_t>(batch) * kQImageBytes, 256) : 0;
  const size_t qs_bytes = w.half_parts ? align_up(static_cast<size_t>(batch) * kQiHeads * sizeof(float), 256) : 0;
  if (base) {
    char* c = static_cast<char*>(base);
    w.part_o = reinterpret_cast<float*>(c);
    w.part_h = reinterpret_cast<uint16_t*>(c);
    w.part_ml = reinterpret_cast<float*>(c + o_bytes);
    w.rope = reinterpret_cast<double*>(c + o_bytes + ml_bytes);
    w.part_sc = reinterpret_cast<float*>(c + o_bytes + ml_bytes + rope_bytes);
    if (w.half_parts) {
      w.qimage = reinterpret_cast<uint8_t*>(c + o_bytes + ml_bytes + rope_bytes + sc_bytes);
      w.qscale = reinterpret_cast<float*>(c + o_bytes + ml_bytes + rope_bytes + sc_bytes + qi_bytes);
    }
  }
  w.bytes = o_bytes + ml_bytes + rope_bytes + sc_bytes + qi_bytes + qs_bytes;
  return w;
}

cudaError_t launch_attention(const LayerParams& p, int batch, const int32_t* seq_len,
                             int max_seq_len, const float* q, const int32_t* idx,
                             const int32_t* cnt, int idx_stride, float* out, const AttnWs& ws,
                             uint32_t* status, cudaStream_t stream, bool prep_done, bool early) {
  cudaError_t e = cudaSuccess;
  if (!prep_done && !attention_tc_supported(p)) {  // the tensor-core kernel writes the table itself
    e = launch_kernel(attn_prep_kernel, dim3(1, batch), dim3(kPrepThreads), 0, stream, p, seq_len, max_seq_len,
                      q, ws);
    if (e != cudaSuccess) return e;
  }
  prof_begin(kProfAttention, stream);
  if (attention_tc_supported(p)) {
    e = launch_attention_tc(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream, early,
                            prep_done);
  } else {
    switch (p.D) {
      case 64: e = launch_simt_d<64>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream); break;
      case 128: e = launch_simt_d<128>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream); break;
      case 256: e = launch_simt_d<256>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream); break;
      case 512: e = launch_simt_d<512>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream); break;
      case 1024: e = launch_simt_d<1024>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream); break;
      default: return cudaErrorInvalidValue;
    }
  }
  if (e != cudaSuccess) return e;
  dim3 grid(p.H, batch);
  if (ws.half_parts) {   // tensor-core path: H = 64, D = 512
    // four split groups per CTA when the requests have many splits (with fewer, most of the
    // groups would idle in the CTAs of short requests)
    const bool many = ws.splits > 2 * kGBatch;
    auto kern = many ? attn_combine_tc_kernel<4, kGBatchMany> : attn_combine_tc_kernel<1, kGBatch>;
    e = launch_kernel(kern, dim3(kGDim / kGDimsPerCta, batch), dim3(many ? 512 : 128), 0, stream, p,
                      seq_len, max_seq_len, cnt, idx != nullptr, idx_stride, ws, out, status, prep_done);
  } else {
    const dim3 block(p.D / 2);   // one thread per pair of dims: 32 .. 512
    e = launch_kernel(attn_combine_kernel, grid, block, 0, stream, p, seq_len, max_seq_len, cnt,
                      idx != nullptr, idx_stride, ws, out, status);
  }
  prof_end(kProfAttention, stream);   // the attention step: its kernel and the split combine
  return e;
}

}  // namespace ckv
