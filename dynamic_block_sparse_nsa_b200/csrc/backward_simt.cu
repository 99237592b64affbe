// NSA prefill backward on CUDA cores (fp32 arithmetic, any head dim / group
// size / dtype the ABI accepts).
//
// The loss gradient flows through the three branches, the gates and the
// compression; the forward's selected blocks are constants (the top-n choice
// is discrete, and the compressed branch is the one that carries the gradient
// that trains selection: EP94 notes §五, branch one; lchairun.cn NSA article,
// the paragraph on trainability). Per query head h of a GQA group and branch c
// with keys k_a, values v_a and probabilities p = softmax(scale q . k_a):
//   dO_c = g_c dO,  D = dO_c . o_c,  dS_a = p_a (dO_c . v_a - D),
//   dq += scale sum_a dS_a k_a,  dk_a += scale dS_a q,  dv_a += p_a dO_c,
// and through the gates g_c = sigmoid(q . Wg[:, c]):
//   dz_c = (dO . o_c) g_c (1 - g_c),  dq += Wg dz,  dWg += q dz^T.
// The compressed keys are K~[i] = sum_j w[j] K[i s + j] (their storage rounding
// taken as the identity), so dK[i s + j] += w[j] dK~[i] and
// dw[j] = sum dK~[i] . K[i s + j] + dV~[i] . V[i s + j].
//
// Launches: bwd_rows (one CTA per (token, KV head): both passes of each branch
// over keys staged through shared memory, dq of the group's heads, dk/dv and
// dK~/dV~ by fp32 atomics, dz to the workspace), bwd_compress (dk, dv += the
// compressed branch's share, a gather per element), bwd_dw (one CTA per
// compression weight), bwd_dwg (one CTA per head-dim index).
#include <algorithm>

#include "device_common.cuh"
#include "internal.h"

namespace nsa {
namespace {

constexpr int kBT = 256;         // threads of bwd_rows
constexpr int kBW = kBT / 32;
constexpr int kBC = 32;          // keys per staged chunk
constexpr int kBwdMaxSel = 64;   // top_n bound (ABI)

struct BwdSmem {
  float* qs;    // [G][d]
  float* dos;   // [G][d]
  float* dqa;   // [G][d] dq accumulator
  float* o;     // [G][d] branch output
  float* Ks;    // [kBC][d + 1]
  float* Vs;    // [kBC][d + 1]
  float* z;     // [G][kBC] logits, then probabilities
  float* ds;    // [G][kBC]
  float* m;     // [G] running max
  float* ls;    // [G] running sum, then lse
  float* fac;   // [G]
  float* D;     // [G]
  float* gt;    // [G][3] gates
  float* dg;    // [G][3] dO . o_c
  int* sel;     // [kBwdMaxSel] valid selected blocks, ascending
  int* misc;    // [4]: number of selected blocks, selected keys
};

__host__ __device__ inline size_t bwd_smem_bytes(int G, int d) {
  const size_t f = 4 * (size_t)G * d + 2 * (size_t)kBC * (d + 1) + 2 * (size_t)G * kBC + 4 * G +
                   6 * (size_t)G;
  return (f + kBwdMaxSel + 4) * 4;
}

__device__ inline BwdSmem carve_bwd(float* p, int G, int d) {
  BwdSmem c;
  c.qs = p; p += G * d;
  c.dos = p; p += G * d;
  c.dqa = p; p += G * d;
  c.o = p; p += G * d;
  c.Ks = p; p += kBC * (d + 1);
  c.Vs = p; p += kBC * (d + 1);
  c.z = p; p += G * kBC;
  c.ds = p; p += G * kBC;
  c.m = p; p += G;
  c.ls = p; p += G;
  c.fac = p; p += G;
  c.D = p; p += G;
  c.gt = p; p += 3 * G;
  c.dg = p; p += 3 * G;
  c.sel = reinterpret_cast<int*>(p);
  c.misc = c.sel + kBwdMaxSel;
  return c;
}

template <typename T>
__global__ void __launch_bounds__(kBT) bwd_rows_kernel(const NsaBwdArgs a) {
  extern __shared__ __align__(16) float bsm[];
  const int G = a.Hq / a.Hkv, d = a.d;
  BwdSmem c = carve_bwd(bsm, G, d);
  const int row = blockIdx.x, g = blockIdx.y;
  const int b = row / a.T, t = row - b * a.T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T* q = static_cast<const T*>(a.q);
  const T* dout = static_cast<const T*>(a.dout);
  const long qrow = ((long)b * a.T + t) * a.Hq + (long)g * G;  // first head of the group

  for (int x = tid; x < G * d; x += kBT) {
    c.qs[x] = to_f32(q[qrow * d + x]);
    c.dos[x] = to_f32(dout[qrow * d + x]);
    c.dqa[x] = 0.f;
  }
  if (tid == 0) {
    // the valid selected blocks (0 <= j <= t / bs), distinct and ascending, so
    // only the last can be the partial block holding t; the keys of the
    // selected branch are their tokens up to t
    const int32_t* srow = a.sel + (((long)b * a.T + t) * a.Hkv + g) * a.n;
    int ns = 0;
    for (int i = 0; i < a.n && i < kBwdMaxSel; ++i) {
      const int j = srow[i];
      if (j < 0 || j > t / a.bs) continue;
      bool seen = false;  // a repeated block counts once
      for (int u = 0; u < ns; ++u) seen |= c.sel[u] == j;
      if (seen) continue;
      int at = ns++;
      while (at > 0 && c.sel[at - 1] > j) {  // insertion keeps the list ascending
        c.sel[at] = c.sel[at - 1];
        --at;
      }
      c.sel[at] = j;
    }
    int nk = 0;
    for (int i = 0; i < ns; ++i) nk += min(a.bs, t + 1 - c.sel[i] * a.bs);
    c.misc[0] = ns;
    c.misc[1] = nk;
  }
  __syncthreads();
  // gates from the raw query: a warp per (head, branch)
  for (int x = warp; x < 3 * G; x += kBW) {
    const int h = x / 3, br = x - 3 * h;
    float gv;
    if (a.gate_mode == 1) {
      gv = a.fixed_gates[br];
    } else {
      float dot = 0.f;
      for (int e = lane; e < d; e += 32) dot = fmaf(c.qs[h * d + e], a.w_gate[e * 3 + br], dot);
      dot = warp_sum(dot);
      gv = 1.f / (1.f + expf(-dot));
    }
    if (lane == 0) c.gt[x] = gv;
  }

  const int nvis = t + 1 >= a.l ? min(a.Nc, (t + 1 - a.l) / a.s + 1) : 0;
  const int w0 = max(0, t - a.w + 1);
  const int nwin = t - w0 + 1;
  const T* kc = static_cast<const T*>(a.kc);
  const T* vc = static_cast<const T*>(a.vc);
  const T* kk = static_cast<const T*>(a.k);
  const T* vv = static_cast<const T*>(a.v);
  const long tok = (long)a.Hkv * d;  // row stride of k, v, k~, v~

  for (int br = 0; br < 3; ++br) {
    __syncthreads();
    const int nk = br == 0 ? nvis : (br == 1 ? c.misc[1] : nwin);
    if (nk == 0) {  // no keys: o_c = 0, nothing to propagate
      for (int h = tid; h < G; h += kBT) c.dg[h * 3 + br] = 0.f;
      continue;
    }
    const T* Kb = br == 0 ? kc + (long)b * a.Nc * tok : kk + (long)b * a.T * tok;
    const T* Vb = br == 0 ? vc + (long)b * a.Nc * tok : vv + (long)b * a.T * tok;
    float* dKb = br == 0 ? a.dkc + (long)b * a.Nc * tok : a.dk + (long)b * a.T * tok;
    float* dVb = br == 0 ? a.dvc + (long)b * a.Nc * tok : a.dv + (long)b * a.T * tok;
    // key a of the branch -> its row in the source
    auto key_row = [&](int ka) {
      if (br == 0) return ka;
      if (br == 1) return c.sel[ka / a.bs] * a.bs + ka % a.bs;
      return w0 + ka;
    };
    auto stage = [&](int c0, int nc) {
      for (int x = tid; x < nc * d; x += kBT) {
        const int col = x / d, e = x - col * d;
        const long r = (long)key_row(c0 + col) * tok + (long)g * d + e;
        c.Ks[col * (d + 1) + e] = to_f32(Kb[r]);
        c.Vs[col * (d + 1) + e] = to_f32(Vb[r]);
      }
    };
    for (int x = tid; x < G * d; x += kBT) c.o[x] = 0.f;
    for (int h = tid; h < G; h += kBT) {
      c.m[h] = -INFINITY;
      c.ls[h] = 0.f;
    }
    // pass 1: softmax statistics and o_c
    for (int c0 = 0; c0 < nk; c0 += kBC) {
      const int nc = min(kBC, nk - c0);
      __syncthreads();
      stage(c0, nc);
      __syncthreads();
      for (int x = tid; x < G * kBC; x += kBT) {
        const int h = x / kBC, col = x - h * kBC;
        if (col < nc) {
          float acc = 0.f;
          for (int e = 0; e < d; ++e) acc = fmaf(c.qs[h * d + e], c.Ks[col * (d + 1) + e], acc);
          c.z[x] = acc * a.scale;
        }
      }
      __syncthreads();
      for (int h = warp; h < G; h += kBW) {
        float* zh = c.z + h * kBC;
        const float zc = lane < nc ? zh[lane] : -INFINITY;  // kBC == 32
        const float mo = c.m[h], mn = fmaxf(mo, warp_max(zc));
        const float pz = lane < nc ? expf(zc - mn) : 0.f;
        if (lane < nc) zh[lane] = pz;
        const float ps = warp_sum(pz);
        if (lane == 0) {
          const float f = expf(mo - mn);  // 0 on the first chunk (mo = -inf)
          c.m[h] = mn;
          c.ls[h] = c.ls[h] * f + ps;
          c.fac[h] = f;
        }
      }
      __syncthreads();
      for (int x = tid; x < G * d; x += kBT) {
        const int h = x / d, e = x - h * d;
        float acc = c.o[x] * c.fac[h];
        for (int col = 0; col < nc; ++col) acc = fmaf(c.z[h * kBC + col], c.Vs[col * (d + 1) + e], acc);
        c.o[x] = acc;
      }
    }
    __syncthreads();
    for (int x = tid; x < G * d; x += kBT) c.o[x] /= c.ls[x / d];
    __syncthreads();
    // dL/dg_c = dO . o_c; D = g_c dO . o_c; lse
    for (int h = warp; h < G; h += kBW) {
      float dot = 0.f;
      for (int e = lane; e < d; e += 32) dot = fmaf(c.dos[h * d + e], c.o[h * d + e], dot);
      dot = warp_sum(dot);
      if (lane == 0) {
        c.dg[h * 3 + br] = dot;
        c.D[h] = c.gt[h * 3 + br] * dot;
        c.ls[h] = c.m[h] + logf(c.ls[h]);
      }
    }
    // pass 2: probabilities again, dS, and the gradients
    for (int c0 = 0; c0 < nk; c0 += kBC) {
      const int nc = min(kBC, nk - c0);
      __syncthreads();
      stage(c0, nc);
      __syncthreads();
      for (int x = tid; x < G * kBC; x += kBT) {
        const int h = x / kBC, col = x - h * kBC;
        if (col < nc) {
          float s = 0.f, dpv = 0.f;
          for (int e = 0; e < d; ++e) {
            s = fmaf(c.qs[h * d + e], c.Ks[col * (d + 1) + e], s);
            dpv = fmaf(c.dos[h * d + e], c.Vs[col * (d + 1) + e], dpv);
          }
          const float pr = expf(s * a.scale - c.ls[h]);
          c.z[x] = pr;
          c.ds[x] = pr * (c.gt[h * 3 + br] * dpv - c.D[h]);
        } else {
          c.z[x] = 0.f;
          c.ds[x] = 0.f;
        }
      }
      __syncthreads();
      // dq of each head; dk, dv of each key summed over the group's heads
      for (int x = tid; x < G * d; x += kBT) {
        const int h = x / d, e = x - h * d;
        float acc = 0.f;
        for (int col = 0; col < nc; ++col) acc = fmaf(c.ds[h * kBC + col], c.Ks[col * (d + 1) + e], acc);
        c.dqa[x] += a.scale * acc;
      }
      for (int x = tid; x < nc * d; x += kBT) {
        const int col = x / d, e = x - col * d;
        float dkv = 0.f, dvv = 0.f;
        for (int h = 0; h < G; ++h) {
          dkv = fmaf(c.ds[h * kBC + col], c.qs[h * d + e], dkv);
          dvv = fmaf(c.z[h * kBC + col] * c.gt[h * 3 + br], c.dos[h * d + e], dvv);
        }
        const long r = (long)key_row(c0 + col) * tok + (long)g * d + e;
        atomicAdd(dKb + r, a.scale * dkv);
        atomicAdd(dVb + r, dvv);
      }
    }
  }
  __syncthreads();
  // gates: dz_c = (dO . o_c) g_c (1 - g_c); dq += Wg dz; dz kept for dWg
  if (a.gate_mode == 0) {
    for (int x = tid; x < G * d; x += kBT) {
      const int h = x / d, e = x - h * d;
      float acc = 0.f;
      for (int br = 0; br < 3; ++br) {
        const float gv = c.gt[h * 3 + br];
        acc = fmaf(a.w_gate[e * 3 + br], c.dg[h * 3 + br] * gv * (1.f - gv), acc);
      }
      c.dqa[x] += acc;
    }
    for (int x = tid; x < G * 3; x += kBT) {
      const float gv = c.gt[x];
      a.dz[qrow * 3 + x] = c.dg[x] * gv * (1.f - gv);
    }
  }
  __syncthreads();
  for (int x = tid; x < G * d; x += kBT) a.dq[qrow * d + x] = c.dqa[x];
}

// dk, dv += the compressed branch's share: element (b, u, g, e) gathers
// w[u - i s] dK~[b, i, g, e] over the compressed blocks i that contain token u.
__global__ void __launch_bounds__(256) bwd_compress_kernel(const NsaBwdArgs a) {
  const long total = (long)a.B * a.T * a.Hkv * a.d;
  const long tok = (long)a.Hkv * a.d;
  for (long x = blockIdx.x * (long)blockDim.x + threadIdx.x; x < total;
       x += (long)gridDim.x * blockDim.x) {
    const long bu = x / tok, ge = x - bu * tok;
    const int b = (int)(bu / a.T), u = (int)(bu - (long)b * a.T);
    const int lo = u - a.l + 1 > 0 ? (u - a.l + 1 + a.s - 1) / a.s : 0;
    const int hi = min(a.Nc - 1, u / a.s);
    float sk = 0.f, sv = 0.f;
    for (int i = lo; i <= hi; ++i) {
      const float wj = a.w_cmp[u - i * a.s];
      const long src = ((long)b * a.Nc + i) * tok + ge;
      sk = fmaf(wj, a.dkc[src], sk);
      sv = fmaf(wj, a.dvc[src], sv);
    }
    a.dk[x] += sk;
    a.dv[x] += sv;
  }
}

template <int NT>
__device__ inline float block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < NT / 32; ++w) s += red[w];
  __syncthreads();
  return s;  // valid in thread 0
}

// dw[j] = sum over (b, i, g, e) of dK~ . K[i s + j] + dV~ . V[i s + j].
template <typename T>
__global__ void __launch_bounds__(256) bwd_dw_kernel(const NsaBwdArgs a) {
  __shared__ float red[8];
  const int j = blockIdx.x;
  const long tok = (long)a.Hkv * a.d;
  const long total = (long)a.B * a.Nc * tok;
  const T* kk = static_cast<const T*>(a.k);
  const T* vv = static_cast<const T*>(a.v);
  float acc = 0.f;
  for (long x = threadIdx.x; x < total; x += blockDim.x) {
    const long bi = x / tok, ge = x - bi * tok;
    const int b = (int)(bi / a.Nc), i = (int)(bi - (long)b * a.Nc);
    const long src = ((long)b * a.T + (long)i * a.s + j) * tok + ge;
    acc = fmaf(a.dkc[x], to_f32(kk[src]), acc);
    acc = fmaf(a.dvc[x], to_f32(vv[src]), acc);
  }
  const float s = block_sum<256>(acc, red);
  if (threadIdx.x == 0) a.dw_cmp[j] = s;
}

// dWg[e][c] = sum over (b, t, h) of q[b, t, h, e] dz[b, t, h, c].
template <typename T>
__global__ void __launch_bounds__(256) bwd_dwg_kernel(const NsaBwdArgs a) {
  __shared__ float red[8];
  const int e = blockIdx.x;
  const long rows = (long)a.B * a.T * a.Hq;
  const T* q = static_cast<const T*>(a.q);
  float acc[3] = {0.f, 0.f, 0.f};
  for (long r = threadIdx.x; r < rows; r += blockDim.x) {
    const float qe = to_f32(q[r * a.d + e]);
    for (int c = 0; c < 3; ++c) acc[c] = fmaf(qe, a.dz[r * 3 + c], acc[c]);
  }
  for (int c = 0; c < 3; ++c) {
    const float s = block_sum<256>(acc[c], red);
    if (threadIdx.x == 0) a.dw_gate[e * 3 + c] = s;
  }
}

template <typename T>
cudaError_t launch_typed(const NsaBwdArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  const size_t smem = bwd_smem_bytes(G, a.d);
  cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    TraceScope trace("bwd_rows", stream);
    bwd_rows_kernel<T><<<dim3((unsigned)(a.B * a.T), (unsigned)a.Hkv), kBT, smem, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.Nc > 0) {
    const long total = (long)a.B * a.T * a.Hkv * a.d;
    const int grid = (int)std::min<long>((total + 255) / 256, 65535L * 8);
    {
      TraceScope trace("bwd_compress", stream);
      bwd_compress_kernel<<<grid, 256, 0, stream>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    TraceScope trace("bwd_dw", stream);
    bwd_dw_kernel<T><<<a.l, 256, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if ((e = cudaMemsetAsync(a.dw_cmp, 0, sizeof(float) * a.l, stream)) != cudaSuccess) {
    return e;
  }
  if (a.gate_mode == 0) {
    TraceScope trace("bwd_dwg", stream);
    bwd_dwg_kernel<T><<<a.d, 256, 0, stream>>>(a);
    return cudaGetLastError();
  }
  return a.dw_gate ? cudaMemsetAsync(a.dw_gate, 0, sizeof(float) * a.d * 3, stream) : cudaSuccess;
}

}  // namespace

size_t nsa_bwd_smem(int G, int d) { return bwd_smem_bytes(G, d); }

size_t nsa_bwd_ws_bytes(const nsa_params& p) {
  const int Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  const size_t cmp = (size_t)p.B * Nc * p.Hkv * p.d * sizeof(float);
  const size_t dz = (size_t)p.B * p.T * p.Hq * 3 * sizeof(float);
  return 2 * ((cmp + 255) & ~size_t(255)) + ((dz + 255) & ~size_t(255));
}

cudaError_t launch_nsa_backward(NsaBwdArgs a, void* ws, cudaStream_t stream) {
  const size_t cmp = ((size_t)a.B * a.Nc * a.Hkv * a.d * sizeof(float) + 255) & ~size_t(255);
  char* w = static_cast<char*>(ws);
  a.dkc = reinterpret_cast<float*>(w);
  a.dvc = reinterpret_cast<float*>(w + cmp);
  a.dz = reinterpret_cast<float*>(w + 2 * cmp);
  const size_t tokb = (size_t)a.B * a.T * a.Hkv * a.d * sizeof(float);
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.dk, 0, tokb, stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dv, 0, tokb, stream)) != cudaSuccess) return e;
  if (cmp > 0 && (e = cudaMemsetAsync(ws, 0, 2 * cmp, stream)) != cudaSuccess) return e;
  return a.dtype == NSA_DTYPE_BF16 ? launch_typed<__nv_bfloat16>(a, stream)
                                   : launch_typed<float>(a, stream);
}

}  // namespace nsa
