// mqa.cu -- shared-KV multi-query attention with sliding window and attention
// sink ("DeepSeek-V4 内部机制" 1.2 Step 2 "Shared-KV MQA", 1.3 HCA dense
// attention, 1.4 window branch and sink equation; yunpan.plus eq. 9).
//
// Every head of a query attends the same rows (the selected compressed
// entries, or all visible entries for HCA, followed by the window tokens) and
// each row serves as both key and value.  The row list of a query is split
// across CTAs (split-KV); each CTA keeps an online softmax per head and writes
// an unnormalised partial (m, l, o); a combine kernel merges the partials in
// split order (deterministic) and adds the sink to the denominator.  With one
// split the CTA finishes the softmax itself.
//
// This file holds the SIMT kernel (fp32 FMA): it serves F32 mode (1e-5
// parity) and every shape the tensor-core kernel (mqa_umma.cu) does not take.
#include "csa_internal.cuh"
#include "mqa_plan.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_mqa)

namespace {

constexpr int kRC = 32;  // rows per chunk (one per lane)

__global__ void __launch_bounds__(256) mqa_simt_kernel(MqaArgs a, MqaPlan plan) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int split = blockIdx.x, hg = blockIdx.y;
  const int64_t bt = blockIdx.z;
  const int b = (int)(bt / a.n_q);
  const int HG = plan.heads_per_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = hg * HG + warp;
  const int dim = a.dim;
  const int stride = dim + 1;  // padded kv rows: lane r reads row r conflict-free

  float* q = reinterpret_cast<float*>(smem_raw);  // [HG][dim]
  float* kv = q + HG * dim;                        // [kRC][dim+1]

  const int64_t t = a.q_pos[bt];
  const RowList rl = make_row_list(a, bt, t);
  const int64_t r_begin = (int64_t)split * plan.rows_per_split;
  const int64_t r_end = min64(rl.n_rows, r_begin + plan.rows_per_split);

  // query heads of this CTA in fp32
  for (int i = threadIdx.x; i < HG * dim; i += blockDim.x) {
    const int hh = i / dim, d = i % dim;
    const int64_t off = (bt * a.n_heads + hg * HG + hh) * dim + d;
    q[i] = a.q_dt == CSA_F32 ? static_cast<const float*>(a.Q)[off]
                             : bf16_bits_to_float(static_cast<const uint16_t*>(a.Q)[off]);
  }

  const int per_lane = dim / 32;
  float o[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const int64_t rb = row_bytes(a.kv_dt, dim);

  for (int64_t c0 = r_begin; c0 < r_end; c0 += kRC) {
    const int nr = (int)min64(kRC, r_end - c0);
    __syncthreads();
    // decode the chunk's rows into shared memory (invalid rows -> zeros)
    for (int i = threadIdx.x; i < kRC * (dim / 8); i += blockDim.x) {
      const int r = i / (dim / 8), d0 = (i % (dim / 8)) * 8;
      float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (r < nr) {
        const uint8_t* src = row_ptr(a, rl, b, c0 + r, rb);
        if (src) decode_row_chunk8(src, nullptr, a.kv_dt, dim, d0, v);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) kv[r * stride + d0 + j] = v[j];
    }
    __syncthreads();
    // logits: lane r scores row c0 + r for head h
    float z = -INFINITY;
    if (lane < nr && row_valid(a, rl, b, c0 + lane)) {
      const float* qh = q + warp * dim;
      const float* kr = kv + lane * stride;
      float dot = 0.f;
      for (int d = 0; d < dim; ++d) dot = fmaf(qh[d], kr[d], dot);
      z = dot * a.scale;
    }
    float cmax = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
    const float m_new = fmaxf(m_run, cmax);
    float p = 0.f, corr = 1.f;
    if (m_new != -INFINITY) {
      p = (z == -INFINITY) ? 0.f : expf(z - m_new);
      corr = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
    }
    float psum = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l_run = l_run * corr + psum;
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j] *= corr;
    for (int r = 0; r < nr; ++r) {
      const float pr = __shfl_sync(0xffffffffu, p, r);
      const float* kr = kv + r * stride;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < per_lane) o[j] = fmaf(pr, kr[lane + 32 * j], o[j]);
    }
  }

  if (plan.n_splits == 1) {
    const float sink = a.sink[h];
    float M = fmaxf(m_run, sink);
    float f = 0.f;
    if (!(sink == INFINITY) && M != -INFINITY) {
      const float em = (m_run == -INFINITY) ? 0.f : expf(m_run - M);
      const float den = l_run * em + expf(sink - M);
      f = em / den;
    }
    const int64_t ob = (bt * a.n_heads + h) * dim;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < per_lane) {
        const float v = o[j] * f;
        if (a.q_dt == CSA_F32) static_cast<float*>(a.O)[ob + lane + 32 * j] = v;
        else static_cast<__nv_bfloat16*>(a.O)[ob + lane + 32 * j] = __float2bfloat16_rn(v);
      }
    }
  } else {
    float* po = plan_partial_o(plan, a, bt, split, h);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < per_lane) po[lane + 32 * j] = o[j];
    if (lane == 0) {
      float* ml = plan_partial_ml(plan, a, bt, split, h);
      ml[0] = m_run;
      ml[1] = l_run;
    }
  }
}

}  // namespace

// Merges the split partials of one (query, head) in split order and applies
// the sink: O = sum_s e^{m_s-M} o_s / (sum_s e^{m_s-M} l_s + e^{sink-M}).
//
// The per-split weights e^{m_s-M}/den are computed once into shared memory
// (kMaxCombineSplits of them; more splits loop over chunks of partials), then
// every thread sums its output dims over the splits with independent loads.
constexpr int kMaxCombineSplits = 256;

__global__ void __launch_bounds__(128) mqa_combine_kernel(MqaArgs a, MqaPlan plan) {
  __shared__ float wgt[kMaxCombineSplits];
  __shared__ float red[4];
  const int h = blockIdx.x;
  const int64_t bt = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float sink = a.sink[h];
  const int S = plan.n_splits;
  // M = max(sink, m_s)
  float M = sink;
  for (int s = threadIdx.x; s < S; s += 128) M = fmaxf(M, plan_partial_ml(plan, a, bt, s, h)[0]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  const bool zero = (sink == INFINITY) || (M == -INFINITY);
  // den = e^{sink-M} + sum_s l_s e^{m_s-M}, summed in split order by one warp
  if (warp == 0) {
    float den = 0.f;
    if (!zero) {
      for (int s0 = 0; s0 < S; s0 += 32) {
        const int s = s0 + lane;
        float v = 0.f;
        if (s < S) {
          const float* ml = plan_partial_ml(plan, a, bt, s, h);
          v = ml[0] == -INFINITY ? 0.f : ml[1] * expf(ml[0] - M);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        den += v;
      }
      den += expf(sink - M);
    }
    if (lane == 0) red[0] = den;
  }
  __syncthreads();
  const float den = red[0];
  const int64_t ob = (bt * a.n_heads + h) * a.dim;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // dims threadIdx.x + 128 j (dim <= 512)
  for (int c0 = 0; c0 < S; c0 += kMaxCombineSplits) {
    const int cn = min(kMaxCombineSplits, S - c0);
    __syncthreads();
    for (int s = threadIdx.x; s < cn; s += 128) {
      const float* ml = plan_partial_ml(plan, a, bt, c0 + s, h);
      wgt[s] = (zero || ml[0] == -INFINITY) ? 0.f : expf(ml[0] - M) / den;
    }
    __syncthreads();
    // splits in groups of 4 so that 16 independent loads are in flight
    int s = 0;
    for (; s + 4 <= cn; s += 4) {
      float v[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* po = plan_partial_o(plan, a, bt, c0 + s + u, h);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int d = threadIdx.x + 128 * j;
          v[u][j] = d < a.dim ? po[d] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(wgt[s + u], v[u][j], acc[j]);
    }
    for (; s < cn; ++s) {
      const float* po = plan_partial_o(plan, a, bt, c0 + s, h);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = threadIdx.x + 128 * j;
        if (d < a.dim) acc[j] = fmaf(wgt[s], po[d], acc[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int d = threadIdx.x + 128 * j;
    if (d >= a.dim) continue;
    if (a.q_dt == CSA_F32) static_cast<float*>(a.O)[ob + d] = acc[j];
    else static_cast<__nv_bfloat16*>(a.O)[ob + d] = __float2bfloat16_rn(acc[j]);
  }
}

// The same merge for few splits (decode on the tensor-core path): thread t
// owns dims 4t .. 4t+3 and loads every split's statistics and partial at
// once, so the kernel waits on one round of loads; the weights are summed in
// split order.
constexpr int kFewSplits = 16;

__global__ void __launch_bounds__(128) mqa_combine_few_kernel(MqaArgs a, MqaPlan plan) {
  const int h = blockIdx.x;
  const int64_t bt = blockIdx.y;
  const int S = plan.n_splits;
  const int d = 4 * threadIdx.x;
  const bool on = d < a.dim;
  float2 ml[kFewSplits];
  float4 o[kFewSplits];
#pragma unroll
  for (int s = 0; s < kFewSplits; ++s)
    if (s < S) {
      ml[s] = __ldcg(reinterpret_cast<const float2*>(plan_partial_ml(plan, a, bt, s, h)));
      o[s] = on ? __ldcg(reinterpret_cast<const float4*>(plan_partial_o(plan, a, bt, s, h) + d))
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  const float sink = a.sink[h];
  float M = sink;
#pragma unroll
  for (int s = 0; s < kFewSplits; ++s)
    if (s < S) M = fmaxf(M, ml[s].x);
  const bool zero = (sink == INFINITY) || (M == -INFINITY);
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < kFewSplits; ++s)
    if (s < S) {
      ml[s].x = (zero || ml[s].x == -INFINITY) ? 0.f : expf(ml[s].x - M);  // e^{m_s - M}
      den += ml[s].x > 0.f ? ml[s].y * ml[s].x : 0.f;
    }
  if (!zero) den += expf(sink - M);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kFewSplits; ++s)
    if (s < S) {
      const float w = zero ? 0.f : ml[s].x / den;
      acc.x = fmaf(w, o[s].x, acc.x);
      acc.y = fmaf(w, o[s].y, acc.y);
      acc.z = fmaf(w, o[s].z, acc.z);
      acc.w = fmaf(w, o[s].w, acc.w);
    }
  if (!on) return;
  const int64_t ob = (bt * a.n_heads + h) * a.dim + d;
  if (a.q_dt == CSA_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(a.O) + ob) = acc;
  } else {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    memcpy(&pk.x, &lo, 4);
    memcpy(&pk.y, &hi, 4);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.O) + ob) = pk;
  }
}

cudaError_t launch_mqa_combine(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  const dim3 grid(a.n_heads, (unsigned)((int64_t)a.batch * a.n_q));
  if (p.n_splits <= kFewSplits && a.dim % 4 == 0 && a.dim <= 512)
    mqa_combine_few_kernel<<<grid, 128, 0, s>>>(a, p);
  else
    mqa_combine_kernel<<<grid, 128, 0, s>>>(a, p);
  ++launch_counter();
  return cudaGetLastError();
}

MqaPlan make_simt_mqa_plan(const MqaArgs& a) {
  MqaPlan p{};
  p.heads_per_cta = (a.n_heads % 8 == 0) ? 8 : (a.n_heads % 4 == 0) ? 4 : (a.n_heads % 2 == 0) ? 2 : 1;
  const int64_t rows_max = max_rows_per_query(a);
  const int64_t units = (int64_t)a.batch * a.n_q * (a.n_heads / p.heads_per_cta);
  // automatic: enough splits to cover the GPU about twice; a fixed count
  // (a.splits) makes the split boundaries depend on the row count only
  int64_t splits = a.splits > 0 ? a.splits : (296 + units - 1) / units;
  const int64_t max_splits = (rows_max + kRC - 1) / kRC;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int64_t rps = (rows_max + splits - 1) / splits;
  rps = (rps + kRC - 1) / kRC * kRC;
  if (rps < kRC) rps = kRC;
  p.rows_per_split = rps;
  p.n_splits = (int)((rows_max + rps - 1) / rps);
  if (p.n_splits < 1) p.n_splits = 1;
  p.mode = p.n_splits > 1 ? kMqaSplit : kMqaWhole;
  p.ws_head = 0;
  return p;
}

cudaError_t launch_mqa_simt(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  const size_t smem = ((size_t)p.heads_per_cta * a.dim + (size_t)kRC * (a.dim + 1)) * 4;
  cudaError_t e = cudaFuncSetAttribute(mqa_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_splits, a.n_heads / p.heads_per_cta, (unsigned)((int64_t)a.batch * a.n_q));
  mqa_simt_kernel<<<grid, 32 * p.heads_per_cta, smem, s>>>(a, p);
  ++launch_counter();
  e = cudaGetLastError();
  if (e != cudaSuccess || p.n_splits == 1) return e;
  return launch_mqa_combine(a, p, s);
}

bool mqa_umma_path(const MqaArgs& a);
MqaPlan mqa_umma_plan(const MqaArgs& a);
cudaError_t launch_mqa_umma(const MqaArgs& a, const MqaPlan& p, cudaStream_t s);

bool mqa_tc_path(const MqaArgs& a) { return mqa_umma_path(a); }

size_t mqa_workspace(const MqaArgs& a) {
  const MqaPlan p = mqa_umma_path(a) ? mqa_umma_plan(a) : make_simt_mqa_plan(a);
  return plan_mqa_workspace_bytes(p, a);
}

cudaError_t launch_mqa(const MqaArgs& a, cudaStream_t s) {
  if (a.has_comp) {
    // the step's entry compression first, on the same stream
    const cudaError_t e = launch_compress(a.comp, s);
    if (e != cudaSuccess) return e;
  }
  if ((int64_t)a.batch * a.n_q == 0) return cudaSuccess;
  if (mqa_umma_path(a)) return launch_mqa_umma(a, mqa_umma_plan(a), s);
  return launch_mqa_simt(a, make_simt_mqa_plan(a), s);
}

}  // namespace csa
