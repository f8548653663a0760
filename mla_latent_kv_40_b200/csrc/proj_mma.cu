// bf16 projections around the attention kernel on warp-level tensor cores.
//
//  * append down-projection [T x D] . [D x (d_c + d_R)] (W_DKV | W_KR), split
//    over D so that every weight element is read once from HBM, then a
//    per-token finish: sum of the splits, RMSNorm of the latent, RoPE of the
//    shared key, scatter into the pool ("DeepSeek-V3 解读 1: MLA", sections
//    "MLA：高层次的思路" and "为什么需要解耦 RoPE");
//  * query absorption q_lat = q_nope . W_UK^(s)T per head plus the RoPE of q_pe
//    ("Transformer升级之路：21、MLA好在哪里?（下）", section 双重投影, decoding column).
// Tiles are 64 rows x 64 or 128 columns, 4 warps of 16 rows each, operands
// staged by cp.async into padded shared tiles and read with ldmatrix.
#include "append_finish.cuh"
#include "kernels.cuh"
#include "mma_tile.cuh"
#include "sm100.cuh"

namespace mla {

using namespace mma;

constexpr int kPT = 128;         // threads per CTA
constexpr int kBM = 64;          // rows (tokens) per CTA
constexpr int kBK = 64;          // K step
constexpr int kPad = 8;          // bf16 elements of padding per smem row

// ------------------------------------------------------------ append: split-K projection
// part[ks][t][n] = sum over k in split ks of h[t][k] * W[k][n], W = [W_DKV | W_KR].
__global__ void __launch_bounds__(kPT)
append_proj_kernel(const __nv_bfloat16 *h, const __nv_bfloat16 *w_dkv, const __nv_bfloat16 *w_kr, int T, int D,
                   int d_c, int d_rope, int k_per_split, float *part) {
  __shared__ __align__(16) __nv_bfloat16 As[2][kBM][kBK + kPad];
  __shared__ __align__(16) __nv_bfloat16 Bs[2][kBK][64 + kPad];
  const int W = d_c + d_rope;
  const int n0 = blockIdx.x * 64;
  const int m0 = blockIdx.y * kBM;
  const int ks = blockIdx.z;
  const int kbeg = ks * k_per_split, kend = min(D, kbeg + k_per_split);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Columns n0..n0+63 lie in one of the two weights (d_c is a multiple of 64).
  const bool in_dkv = n0 < d_c;
  const __nv_bfloat16 *wb = in_dkv ? w_dkv + n0 : w_kr + (n0 - d_c);
  const int ldw = in_dkv ? d_c : d_rope;
  const int ncols = min(64, W - n0);

  auto load = [&](int buf, int k0) {
    // A: 64 rows x 64 k = 512 chunks of 16 B; B: 64 k x 64 n = 512 chunks.
    for (int c = tid; c < 512; c += kPT) {
      const int r = c >> 3, q = c & 7;
      const int t = m0 + r;
      cp16(&As[buf][r][q * 8], h + (int64_t)min(t, T - 1) * D + k0 + q * 8, t < T);
      const int kk = k0 + r;
      cp16(&Bs[buf][r][q * 8], wb + (int64_t)kk * ldw + q * 8, q * 8 < ncols);
    }
    cp_commit();
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  int buf = 0;
  load(0, kbeg);
  for (int k0 = kbeg; k0 < kend; k0 += kBK) {
    if (k0 + kBK < kend) {
      load(buf ^ 1, k0 + kBK);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; kk += 16) {
      uint32_t a[4];
      load_a(&As[buf][0][0], kBK + kPad, warp * 16, kk, a);
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b[4];
        load_b2(&Bs[buf][0][0], 64 + kPad, kk, nt * 8, true, b);
        mma16816(acc[nt], a, b[0], b[1]);
        mma16816(acc[nt + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
    buf ^= 1;
  }
  const int g = lane >> 2, q = lane & 3;
  float *dst = part + (int64_t)ks * T * W;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int col = n0 + nt * 8 + 2 * q;
    if (col >= n0 + ncols) continue;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int t = m0 + warp * 16 + g + 8 * hf;
      if (t < T) *reinterpret_cast<float2 *>(dst + (int64_t)t * W + col) = make_float2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
    }
  }
}

// One CTA per token, one thread per pair of columns: sum the splits (independent loads, so
// they are in flight together), RMSNorm over d_c, RoPE the shared key, scatter.
constexpr int kFinThreads = 288;   // (d_c + d_R) / 2 column pairs of the V3 and V2-Lite rows

__global__ void __launch_bounds__(kFinThreads)
append_finish_kernel(AppendArgs a, const float *part, int nsplit) {
  __shared__ float red[kFinishScratch];
  sm100::grid_dep_launch();
  sm100::grid_dep_wait();   // the partials come from the projection kernel just before
  const int tok = blockIdx.x;
  append_finish_token<kFinThreads>(a, part, nsplit, tok, a.seq_idx[tok], a.pos[tok], red);
}

size_t append_mma_workspace(int T, int d_model, int W, int *nsplit, int *k_per_split) {
  const int mtiles = (T + kBM - 1) / kBM;
  const int ntiles = (W + 63) / 64;
  const int ksteps = d_model / kBK;
  int want = (2 * 148 + ntiles * mtiles - 1) / (ntiles * mtiles);
  want = want < 1 ? 1 : (want > ksteps ? ksteps : want);
  const int steps_per = (ksteps + want - 1) / want;
  const int ns = (ksteps + steps_per - 1) / steps_per;
  if (nsplit) *nsplit = ns;
  if (k_per_split) *k_per_split = steps_per * kBK;
  return (size_t)ns * T * W * sizeof(float);
}

bool append_mma_supported(const AppendArgs &a, bool bf16) {
  return bf16 && a.d_model % kBK == 0 && a.d_c % 64 == 0 && a.d_rope <= 64 && a.d_rope % 8 == 0 &&
         a.d_c + a.d_rope <= 2 * 2 * kFinThreads;
}

int launch_append_mma(const AppendArgs &a, void *ws, cudaStream_t st) {
  int nsplit = 1, kps = a.d_model;
  const int W = a.d_c + a.d_rope;
  append_mma_workspace(a.T, a.d_model, W, &nsplit, &kps);
  float *part = static_cast<float *>(ws);
  const dim3 grid((W + 63) / 64, (a.T + kBM - 1) / kBM, nsplit);
  append_proj_kernel<<<grid, kPT, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.h),
                                           static_cast<const __nv_bfloat16 *>(a.w_dkv),
                                           static_cast<const __nv_bfloat16 *>(a.w_kr), a.T, a.d_model, a.d_c,
                                           a.d_rope, kps, part);
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  return launch_append_finish(a, part, nsplit, st);
}

int launch_append_finish(const AppendArgs &a, const void *ws, int nsplit, cudaStream_t st) {
  return launch_pdl(append_finish_kernel, dim3(a.T), dim3(kFinThreads), 0, st, a, static_cast<const float *>(ws),
                    nsplit) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

// ------------------------------------------------------------ query absorption
// q_out[r][s][n0 + n] = sum_k q_nope[r][s][k] W_UK[s][n0 + n][k], n < 128, plus (z == 0) the
// rotated q_pe.  CTA = (head s, 64 query rows, 128 latent columns); W_UK[s] is [d_c][d_nope].
__global__ void __launch_bounds__(kPT)
absorb_mma_kernel(AbsorbArgs a) {
  extern __shared__ __align__(16) __nv_bfloat16 sm[];
  const int dn = a.d_nope, ld = dn + kPad;
  __nv_bfloat16 *As = sm;                    // [64][dn + pad]
  __nv_bfloat16 *Bs = sm + kBM * ld;         // [128][dn + pad]
  const int s = blockIdx.x, m0 = blockIdx.y * kBM, n0 = blockIdx.z * 128;
  const int R = a.B * a.n_q, W = a.d_c + a.d_rope;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __nv_bfloat16 *qn = static_cast<const __nv_bfloat16 *>(a.q_nope);
  const __nv_bfloat16 *wuk = static_cast<const __nv_bfloat16 *>(a.w_uk) + (int64_t)s * a.d_c * dn;
  const int cpr = dn / 8;                    // 16-byte chunks per row
  for (int c = tid; c < kBM * cpr; c += kPT) {
    const int r = c / cpr, q = c % cpr, gr = m0 + r;
    cp16(As + r * ld + q * 8, qn + ((int64_t)min(gr, R - 1) * a.H + s) * dn + q * 8, gr < R);
  }
  for (int c = tid; c < 128 * cpr; c += kPT) {
    const int n = c / cpr, q = c % cpr;
    cp16(Bs + n * ld + q * 8, wuk + (int64_t)(n0 + n) * dn + q * 8, true);
  }
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int kk = 0; kk < dn; kk += 16) {
    uint32_t af[4];
    load_a(As, ld, warp * 16, kk, af);
#pragma unroll
    for (int nt = 0; nt < 16; nt += 2) {
      uint32_t b[4];
      load_b2(Bs, ld, kk, nt * 8, false, b);
      mma16816(acc[nt], af, b[0], b[1]);
      mma16816(acc[nt + 1], af, b[2], b[3]);
    }
  }
  __nv_bfloat16 *qo = static_cast<__nv_bfloat16 *>(a.q_out);
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int gr = m0 + warp * 16 + g + 8 * hf;
      if (gr < R)
        *reinterpret_cast<__nv_bfloat162 *>(qo + ((int64_t)gr * a.H + s) * W + n0 + nt * 8 + 2 * q) =
            __floats2bfloat162_rn(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
    }
  // RoPE of q_pe, spread over the gridDim.z CTAs of this (head, row tile): CTA z takes rows
  // z, z + gridDim.z, ...; the pair frequencies are computed once per CTA.
  __shared__ double theta[32];
  const int half = a.d_rope / 2;
  if (tid < half) theta[tid] = rope_theta(tid, a.d_rope, a.rope_base);
  __syncthreads();
  const __nv_bfloat16 *qp = static_cast<const __nv_bfloat16 *>(a.q_pe);
  for (int e = tid; e < kBM * half; e += kPT) {
    const int r = blockIdx.z + gridDim.z * (e / half), i = e % half, gr = m0 + r;
    if (r >= kBM || gr >= R) continue;
    const int b = gr / a.n_q, j = gr % a.n_q;
    const int p = a.seqlens[b] - a.n_q + j;
    float cs, sn;
    rope_cos_sin_theta(p < 0 ? 0 : p, theta[i], &cs, &sn);
    const int64_t src = ((int64_t)gr * a.H + s) * a.d_rope + 2 * i;
    const float x = __bfloat162float(qp[src]), y = __bfloat162float(qp[src + 1]);
    *reinterpret_cast<__nv_bfloat162 *>(qo + ((int64_t)gr * a.H + s) * W + a.d_c + 2 * i) =
        __floats2bfloat162_rn(x * cs - y * sn, x * sn + y * cs);
  }
}

bool absorb_mma_supported(const AbsorbArgs &a, bool bf16) {
  return bf16 && a.d_nope % 16 == 0 && a.d_nope <= 256 && a.d_c % 128 == 0 && a.d_rope <= 64;
}

int launch_absorb_mma(const AbsorbArgs &a, cudaStream_t st) {
  const size_t smem = sizeof(__nv_bfloat16) * (kBM + 128) * (a.d_nope + kPad);
  if (cudaFuncSetAttribute(absorb_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
    return MLA_ERR_CUDA;
  const dim3 grid(a.H, (a.B * a.n_q + kBM - 1) / kBM, a.d_c / 128);
  absorb_mma_kernel<<<grid, kPT, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
