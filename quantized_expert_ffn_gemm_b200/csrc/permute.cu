// Token permutation, weighted combine, RMSNorm and the dequantization test hook.
//
// Permutation: the routed (token, slot) pairs are grouped into expert-contiguous rows so each
// expert's rows form one GEMM operand (the more tokens an expert collects in a prefill chunk,
// the more its weights are reused: "Two-Day Port, 8x Faster Prefill: Strata Engine
// Benchmarked", "Where Strata Is Fast: Not Magic, but Logistics", MoE paragraph). It is a
// stable counting sort: per-chunk histograms (stored expert-major, hist[e][chunk]), one
// exclusive scan over (expert, chunk), then a stable scatter in which one warp walks its chunk
// in order and ranks equal experts with __match_any_sync, so the rows of an expert come out in
// token order, deterministically.
#include "common.cuh"
#include "dequant.cuh"

namespace moe {

// ---------------------------------------------------------------- histogram per chunk
__global__ void __launch_bounds__(256)
perm_hist_kernel(const int32_t *__restrict__ idx, int P, int E, int32_t *__restrict__ hist, Ctrl *ctrl) {
  extern __shared__ int32_t sh[];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int p0 = c * kPermChunk;
  for (int p = p0 + threadIdx.x; p < min(P, p0 + kPermChunk); p += blockDim.x) {
    int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&sh[e], 1);
    else set_device_error(ctrl, MOE_ERR_DEVICE_CHECK, e);
  }
  __syncthreads();
  const int nchunks = gridDim.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)e * nchunks + c] = sh[e];
}

// ---------------------------------------------------------------- scan (one CTA)
// counts[e] = sum_c hist[e][c]; offsets = exclusive scan over e; hist[e][c] <- first row of
// chunk c in expert e. The kernel is bound by dependent round trips to memory, so it makes as
// few as it can: a single chunk is read by the scanning threads in one round of loads; a
// histogram that fits in shared memory is staged there in one round and scanned row by row; a
// larger one is walked by warps (one expert per warp at a time, its lanes reading the expert's
// chunk counts and scanning them with shuffles, four experts' loads in flight together).
constexpr size_t kScanSmemMax = 200 * 1024;

__global__ void __launch_bounds__(1024)
perm_scan_kernel(int32_t *__restrict__ hist, int nchunks, int E, int P, int T, int with_shared, int staged,
                 int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
  extern __shared__ int32_t s_cnt[];  // [E] totals, then exclusive offsets; then [E][nchunks] if staged
  __shared__ int32_t s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;  // experts per thread in the scan
  // one chunk (up to kPermChunk pairs): the chunk counts are the totals, read by the scanning
  // threads themselves in one round of loads; the two warp passes below are skipped
  const bool one = nchunks == 1;
  // several chunks, when the whole histogram fits in shared memory (staged): it is copied in with
  // one round of 16-byte loads into rows of an odd stride (32 consecutive experts then fall on 32
  // banks); each thread sums and later prefixes its own experts' rows there, and the prefixes go
  // back with coalesced stores. The warp passes below serve only histograms too large to stage.
  const bool stg = staged && !one;
  const int Pp = nchunks | 1;
  int32_t *s_h = s_cnt + ((E + 3) & ~3);
  auto sidx = [&](int q) { return (q / nchunks) * Pp + q % nchunks; };  // global [e][c] -> shared
  if (stg) {
    const int n = E * nchunks, n4 = n >> 2;
    const int4 *g4 = reinterpret_cast<const int4 *>(hist);
    for (int i0 = tid; i0 < n4; i0 += 8 * (int)blockDim.x) {  // 8 loads in flight per thread
      int4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * (int)blockDim.x;
        v[j] = (i < n4) ? g4[i] : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * (int)blockDim.x;
        if (i < n4) {
          s_h[sidx(4 * i)] = v[j].x;
          s_h[sidx(4 * i + 1)] = v[j].y;
          s_h[sidx(4 * i + 2)] = v[j].z;
          s_h[sidx(4 * i + 3)] = v[j].w;
        }
      }
    }
    for (int q = 4 * n4 + tid; q < n; q += blockDim.x) s_h[sidx(q)] = hist[q];
    __syncthreads();
    for (int i = 0; i < per; ++i) {  // this thread's experts: row totals
      const int e = tid * per + i;
      if (e < E) {
        const int32_t *row = s_h + (size_t)e * Pp;
        int tot = 0;
        for (int c = 0; c < nchunks; ++c) tot += row[c];
        s_cnt[e] = tot;
      }
    }
  }
  // pass 1: per-expert totals, four experts per warp iteration so their loads are in flight together
  for (int e0 = warp; !one && !stg && e0 < E; e0 += 4 * nw) {
    int sum[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * nw;
      sum[u] = 0;
      if (e < E) {
        const int32_t *h = hist + (size_t)e * nchunks;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = lane + 32 * i;
          if (c < nchunks) sum[u] += h[c];
        }
        for (int c = lane + 128; c < nchunks; c += 32) sum[u] += h[c];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int v = sum[u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      const int e = e0 + u * nw;
      if (lane == 0 && e < E) s_cnt[e] = v;
    }
  }
  __syncthreads();
  // exclusive scan of the E totals (contiguous runs per thread, then a block scan of the runs)
  int mysum = 0;
  for (int i = 0; i < per; ++i) {
    const int e = tid * per + i;
    if (e < E) mysum += one ? hist[e] : s_cnt[e];
  }
  int v = mysum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int wv = (lane < nw) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += n;
    }
    s_warp[lane] = wv;
  }
  __syncthreads();
  int base = v - mysum + (warp > 0 ? s_warp[warp - 1] : 0);
  for (int i = 0; i < per; ++i) {
    const int e = tid * per + i;
    if (e < E) {
      const int c = one ? hist[e] : s_cnt[e];
      counts[e] = c;
      offsets[e] = base;
      if (one) {
        hist[e] = base;  // the chunk's first row in expert e
      } else if (stg) {  // first row of every chunk of expert e, in place in its shared row
        int32_t *row = s_h + (size_t)e * Pp;
        int run = base;
        for (int cc = 0; cc < nchunks; ++cc) {
          const int v = row[cc];
          row[cc] = run;
          run += v;
        }
      } else {
        s_cnt[e] = base;  // this thread alone reads and rewrites entry e
      }
      base += c;
    }
  }
  __syncthreads();
  if (stg) {  // the prefixes back to global memory, 16-byte stores
    const int n = E * nchunks, n4 = n >> 2;
    int4 *g4 = reinterpret_cast<int4 *>(hist);
    for (int i = tid; i < n4; i += blockDim.x)
      g4[i] = make_int4(s_h[sidx(4 * i)], s_h[sidx(4 * i + 1)], s_h[sidx(4 * i + 2)], s_h[sidx(4 * i + 3)]);
    for (int q = 4 * n4 + tid; q < n; q += blockDim.x) hist[q] = s_h[sidx(q)];
  }
  // pass 2: first row of every (expert, chunk): the expert's offset + the exclusive prefix over
  // chunks. Four experts per warp iteration, and each expert's chunk counts (up to 128 at a
  // time) are loaded before any is scanned, so a warp has up to 16 loads in flight.
  for (int e0 = warp; !one && !stg && e0 < E; e0 += 4 * nw) {
    int run[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) run[u] = (e0 + u * nw < E) ? s_cnt[e0 + u * nw] : 0;
    for (int c0 = 0; c0 < nchunks; c0 += 128) {
      int xv[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * nw;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = c0 + 32 * i + lane;
          xv[u][i] = (e < E && c < nchunks) ? hist[(size_t)e * nchunks + c] : 0;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * nw;
        if (e >= E) break;  // warp-uniform
        int32_t *h = hist + (size_t)e * nchunks;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = c0 + 32 * i + lane;
          int incl = xv[u][i];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
          }
          if (c < nchunks) h[c] = run[u] + incl - xv[u][i];
          run[u] += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
    }
  }
  if (tid == 0) {
    offsets[E] = P;
    if (with_shared) {
      offsets[E + 1] = P + T;
      counts[E] = T;
    }
  }
}

// ---------------------------------------------------------------- stable scatter (one warp per chunk)
// n_iota > 0: the shared expert's rows, src[P + t] = t for t < n_iota, are written here too
__global__ void __launch_bounds__(32)
perm_scatter_kernel(const int32_t *__restrict__ idx, int P, int k, int E, const int32_t *__restrict__ hist,
                    int32_t *__restrict__ row_of, int32_t *__restrict__ src, int n_iota) {
  extern __shared__ int32_t cursor[];
  const int c = blockIdx.x, lane = threadIdx.x, nchunks = gridDim.x;
  for (int t = c * 32 + lane; t < n_iota; t += nchunks * 32) src[P + t] = t;
  for (int e = lane; e < E; e += 32) cursor[e] = hist[(size_t)e * nchunks + c];
  __syncwarp();
  const int p0 = c * kPermChunk, p1 = min(P, p0 + kPermChunk);
  int ev[kPermChunk / 32];  // the chunk's expert ids, loaded before the in-order walk
#pragma unroll
  for (int i = 0; i < kPermChunk / 32; ++i) {
    const int p = p0 + 32 * i + lane;
    ev[i] = (p < p1) ? idx[p] : -1;
  }
#pragma unroll
  for (int i = 0; i < kPermChunk / 32; ++i) {
    const int pb = p0 + 32 * i;
    if (pb >= p1) break;
    int p = pb + lane;
    int e = ev[i];
    bool ok = (p < p1) && e >= 0 && e < E;
    int key = ok ? e : -1 - lane;  // invalid lanes form singleton groups
    unsigned grp = __match_any_sync(0xffffffffu, key);
    int rank = __popc(grp & ((1u << lane) - 1u));
    int base = ok ? cursor[e] : 0;
    __syncwarp();
    if (ok) {
      int row = base + rank;
      row_of[p] = row;
      src[row] = p / k;
      if (rank == 0) cursor[e] = base + __popc(grp);
    } else if (p < p1) {
      row_of[p] = -1;  // flagged by the histogram kernel
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------- gather rows (bf16 -> fp16)
// one warp per row: the row's 16-byte chunks are all loaded (eight per lane at H = 2048) before
// any is converted and stored, and the warp's next source token is read meanwhile
__global__ void __launch_bounds__(256)
perm_gather_kernel(const uint16_t *__restrict__ x, int H, const int32_t *__restrict__ src, int P, int rows,
                   uint16_t *__restrict__ x_perm, Ctrl *__restrict__ ctrl) {
  const int lane = threadIdx.x & 31, H8 = H >> 3, stride = gridDim.x * 8;
  bool bad = false;  // an x value beyond the fp16 range
  int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  int t = (r < rows) ? ((r < P) ? src[r] : r - P) : 0;
  for (; r < rows; r += stride) {
    // the next row's source token is requested along with this row's data
    const int rn = r + stride;
    const int tn = (rn < rows) ? ((rn < P) ? src[rn] : rn - P) : 0;
    const uint4 *xs = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    uint4 *xd = reinterpret_cast<uint4 *>(x_perm + (size_t)r * H);
    for (int c0 = lane; c0 < H8; c0 += 256) {  // H = 2048: the whole row in one round of loads
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + 32 * u;
        v[u] = (c < H8) ? __ldg(xs + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + 32 * u;
        if (c >= H8) break;
        const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __half2 h = __floats2half2_rn(__uint_as_float(in[j] << 16), __uint_as_float(in[j] & 0xffff0000u));
          out[j] = *reinterpret_cast<uint32_t *>(&h);
          bad |= f16x2_inf(out[j]);
        }
        xd[c] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
    t = tn;
  }
  if (bad) set_device_error(ctrl, MOE_ERR_RANGE, 1);
}

cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, const uint16_t *x, int H, int with_shared,
                           int32_t *counts, int32_t *offsets, int32_t *row_of, int32_t *src, uint16_t *x_perm,
                           int32_t *hist, Ctrl *ctrl, cudaStream_t s) {
  const int P = T * k;
  const int nchunks = (P + kPermChunk - 1) / kPermChunk;
  const size_t esm = (size_t)E * 4;
  {
    KTimer kt_(KID_PERM_HIST, s);
    perm_hist_kernel<<<nchunks, 256, esm, s>>>(idx, P, E, hist, ctrl);
  }
  {
    KTimer kt_(KID_PERM_SCAN, s);
    // the histogram staged in shared memory when it fits (8192 tokens x top-10: 160 KB)
    const size_t hsm = (size_t)E * (nchunks | 1) * 4, esm4 = (size_t)((E + 3) & ~3) * 4;  // odd row stride
    const int staged = (nchunks > 1 && esm4 + hsm <= kScanSmemMax) ? 1 : 0;
    const size_t sm = staged ? esm4 + hsm : esm;
    if (staged) {
      const cudaError_t e = smem_limit_once(perm_scan_kernel, kScanSmemMax);
      if (e != cudaSuccess) return e;
    }
    perm_scan_kernel<<<1, 1024, sm, s>>>(hist, nchunks, E, P, T, with_shared, staged, counts, offsets);
  }
  {
    KTimer kt_(KID_PERM_SCATTER, s);
    perm_scatter_kernel<<<nchunks, 32, esm, s>>>(idx, P, k, E, hist, row_of, src, with_shared ? T : 0);
  }
  const int rows = P + (with_shared ? T : 0);
  size_t want = ((size_t)rows + 7) / 8, cap = (size_t)num_sms() * 16;
  int grid = (int)(want < cap ? want : cap);
  {
    KTimer kt_(KID_PERM_GATHER, s);
    perm_gather_kernel<<<grid, 256, 0, s>>>(x, H, src, P, rows, x_perm, ctrl);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- combine
// y[t,h] = sum_j w[t,j] out[row_of[t,j], h] (fixed j order) + shared[t,h] + residual[t,h]
// One warp per (token, 256-column segment) item, so a small batch still spreads over many warps:
// lanes j < k hold the token's rows and weights (broadcast by shuffle), each lane owns one
// 8-column chunk and issues the k row loads of it before accumulating them.
__global__ void __launch_bounds__(256)
combine_kernel(const uint16_t *__restrict__ out, const int32_t *__restrict__ row_of, const float *__restrict__ w,
               int T, int k, int H, const uint16_t *__restrict__ shared, const float *residual, float *y,
               Ctrl *__restrict__ ctrl) {
  const int lane = threadIdx.x & 31, H8 = H >> 3, nseg = (H8 + 31) >> 5;
  // an expert output outside the fp16 range (an overflowed h gives a non-finite output too): the
  // grouped GEMM's epilogues store without a check, so the range is checked here, once per value
  uint32_t bad = 0;
  const long long n_items = (long long)T * nseg;
  for (long long it = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); it < n_items; it += (long long)gridDim.x * 8) {
    const int t = (int)(it / nseg), c = (int)(it % nseg) * 32 + lane;
    const int my_row = (lane < k) ? row_of[(size_t)t * k + lane] : -1;
    const float my_w = (lane < k) ? w[(size_t)t * k + lane] : 0.0f;
    const bool cok = c < H8;  // every lane stays for the shuffles
    {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
      if (residual && cok) {
        const float4 r0 = reinterpret_cast<const float4 *>(residual + (size_t)t * H)[2 * c];
        const float4 r1 = reinterpret_cast<const float4 *>(residual + (size_t)t * H)[2 * c + 1];
        acc[0] = r0.x; acc[1] = r0.y; acc[2] = r0.z; acc[3] = r0.w;
        acc[4] = r1.x; acc[5] = r1.y; acc[6] = r1.z; acc[7] = r1.w;
      }
      for (int j0 = 0; j0 < k; j0 += 4) {
        uint4 v[4];
        float wj[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rj = __shfl_sync(0xffffffffu, my_row, (j0 + u) & 31);
          wj[u] = __shfl_sync(0xffffffffu, my_w, (j0 + u) & 31);
          const bool use = cok && j0 + u < k && rj >= 0;  // rows past k or flagged (-1) add nothing
          v[u] = use ? __ldg(reinterpret_cast<const uint4 *>(out + (size_t)rj * H) + c) : make_uint4(0, 0, 0, 0);
          if (!use) wj[u] = 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // exponent all ones in either half: inf or NaN
            bad |= ((vv[q] & 0x7c00u) == 0x7c00u) | ((vv[q] & 0x7c000000u) == 0x7c000000u);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&vv[q]));
            acc[2 * q] = fmaf(wj[u], f.x, acc[2 * q]);
            acc[2 * q + 1] = fmaf(wj[u], f.y, acc[2 * q + 1]);
          }
        }
      }
      if (shared && cok) {
        const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(shared + (size_t)t * H) + c);
        const uint32_t vv[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          bad |= ((vv[q] & 0x7c00u) == 0x7c00u) | ((vv[q] & 0x7c000000u) == 0x7c000000u);
          const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&vv[q]));
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      }
      if (cok) {
        float4 *yo = reinterpret_cast<float4 *>(y + (size_t)t * H);
        yo[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yo[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
  if (bad && ctrl) set_device_error(ctrl, MOE_ERR_RANGE, 8);
}

cudaError_t launch_combine(const uint16_t *out_perm, const int32_t *row_of, const float *w, int T, int k, int H,
                           const uint16_t *shared_out, const float *residual, float *y, cudaStream_t s, Ctrl *ctrl) {
  // items of (token, 256-column segment), eight warps per block
  const size_t nseg = ((size_t)(H / 8) + 31) / 32;
  size_t want = ((size_t)T * nseg + 7) / 8, cap = (size_t)num_sms() * 16;
  int grid = (int)(want < cap ? want : cap);
  {
    KTimer kt_(KID_COMBINE, s);
    combine_kernel<<<grid, 256, 0, s>>>(out_perm, row_of, w, T, k, H, shared_out, residual, y, ctrl);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- RMSNorm
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const float *__restrict__ r, int H, float eps, uint16_t *__restrict__ u) {
  __shared__ float s_part[8];
  const int t = blockIdx.x;
  const float *row = r + (size_t)t * H;
  float ss = 0.0f;
  for (int h = threadIdx.x; h < H; h += blockDim.x) ss = fmaf(row[h], row[h], ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += s_part[i];
  const float inv = 1.0f / sqrtf(tot / (float)H + eps);
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    __nv_bfloat16 b = __float2bfloat16_rn(row[h] * inv);
    u[(size_t)t * H + h] = *reinterpret_cast<uint16_t *>(&b);
  }
}

cudaError_t launch_rmsnorm(const float *r, int T, int H, float eps, uint16_t *u, cudaStream_t s) {
  {
    KTimer kt_(KID_RMSNORM, s);
    rmsnorm_kernel<<<T, 256, 0, s>>>(r, H, eps, u);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- dequant test hook
// thread per (row, 16-weight word); fp16 output through the same pair decoder the GEMM uses
__global__ void dequant_rows_kernel(moe_qmat m, int expert, int row0, int nrows, float *out_f32, uint16_t *out_f16) {
  // one code word per thread: 16 weights of the 2-bit plane, 8 of the 4-bit plane
  const bool q4 = m.qtype == MOE_Q4;
  const int per = q4 ? 8 : 16;
  const int words = m.K / per;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nrows * words) return;
  const int r = i / words, wq = i % words;
  const size_t row = (size_t)expert * m.rows + row0 + r;
  const int blk = wq / (32 / per), q = wq % (32 / per);
  const uint32_t w = reinterpret_cast<const uint32_t *>(m.codes + row * (q4 ? m.K / 2 : m.K / 4))[wq];
  const uint16_t dbits = m.scales[row * (m.K / 32) + blk];
  const __half d = __ushort_as_half(dbits);
  uint32_t pairs[8];
  if (m.qtype == MOE_Q2) {
    dq2_word(w, __half2half2(d), pairs);
  } else if (q4) {
    dq4_word(w, __half2half2(d), pairs);
  } else {
    const uint32_t hw = reinterpret_cast<const uint32_t *>(m.hibits + row * (m.K / 8))[blk];
    dq3_word(w, hw, q, __half2half2(d), pairs);
  }
  const float df = __half2float(d);
  const int q0 = (m.qtype == MOE_Q2) ? 2 : q4 ? 8 : 4;
  for (int j = 0; j < per; ++j) {
    const int kk = wq * per + j;
    const uint16_t hb = (uint16_t)((pairs[j >> 1] >> (16 * (j & 1))) & 0xffffu);
    if (out_f16) out_f16[(size_t)r * m.K + kk] = hb;
    if (out_f32) {
      // integer code recovered from the packed planes (independent of the fp16 path)
      const int ii = j >> 1, h = j & 1;
      int c;
      if (q4) {
        c = (int)((w >> (16 * h + 4 * ii)) & 15u);
      } else {
        c = (int)((w >> (16 * h + 2 * ii)) & 3u);
        if (m.qtype == MOE_Q3) {
          const uint32_t hw = reinterpret_cast<const uint32_t *>(m.hibits + row * (m.K / 8))[blk];
          c |= (int)((hw >> (16 * h + 8 * q + ii)) & 1u) << 2;
        }
      }
      out_f32[(size_t)r * m.K + kk] = df * (float)(c - q0);
    }
  }
}

cudaError_t launch_dequant_rows(const moe_qmat &m, int expert, int row0, int nrows, float *out_f32, uint16_t *out_f16,
                                cudaStream_t s) {
  const int n = nrows * (m.K / (m.qtype == MOE_Q4 ? 8 : 16));
  {
    KTimer kt_(KID_DEQUANT_ROWS, s);
    dequant_rows_kernel<<<(n + 255) / 256, 256, 0, s>>>(m, expert, row0, nrows, out_f32, out_f16);
  }
  return cudaGetLastError();
}

}  // namespace moe
