// Decode GEMV for M = 1 (the main decode path): y[n] = sum_k x[k] * w[n][k] + b[n].
//
// The weight stream (0.625 B per weight) is the whole cost. Measured on B200: a plain read
// of the same bytes by many warps with 16-byte loads is the fastest way to pull them in;
// a single bulk-copy producer per SM could not issue fast enough. So every lane loads its
// own codes:
//   * one CTA per SM owns a balanced contiguous range of rows, split again between warp
//     groups; the warps of a group own consecutive 32-column chunks (lane = chunk = one
//     scale group = 16 code bytes), so a warp reads 512 contiguous code bytes and 128
//     contiguous scale bytes per row -- fully coalesced;
//   * each lane keeps its activation chunk in registers for the whole kernel and prefetches
//     the codes and scale of the rows 4 ahead through a register ring (no shared memory on
//     the load path);
//   * math per chunk: one LOP3 per nibble pair (the nibble drops into the mantissa of 128.0,
//     whose ulp is 1), one exact bf16x2 FMA removing the offset, and the sm_100
//     mixed-precision FMA (bf16 x bf16 + fp32, full rate, exact product) in four independent
//     chains; the group scale multiplies the fp32 partial;
//   * every 8 rows the group reduces across lanes (transposing butterfly) and across its
//     warps (shared memory, fixed order: deterministic) and writes y.
// Asymmetric act-order codes (sorted by w4_asym_prepare) take the same path with unsigned
// nibbles minus the row's zero point and x gathered through perm.
#include "w4_dot.cuh"
#include "w4_sync.cuh"

namespace w4i {

namespace {

constexpr int kAhead = 4;  // rows prefetched ahead per lane

struct RowsGeom {
  int64_t P;   // code bytes per row
  int64_t SG;  // scale (and zero) columns per row
  int wg;      // warps per group: ceil(C / 32)
  int ngroups;
  int x_vec;
};

template <bool ASYM>
struct RowData {
  uint4 c;
  float s;
  uint32_t z;
};

template <int NW, bool ASYM>
__global__ void __launch_bounds__(NW * 32, 1) gemv_rows_kernel(const LinearParams p, const RowsGeom g) {
  __shared__ float red[2][NW][kGemvRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / g.wg, wig = warp % g.wg;
  if (grp >= g.ngroups) return;
  const int64_t N = p.N, K = p.K;
  const int64_t C = (K + 31) / 32;
  const int64_t cr0 = static_cast<int64_t>(blockIdx.x) * N / gridDim.x;
  const int64_t cr1 = static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x;
  const int64_t r_begin = cr0 + (cr1 - cr0) * grp / g.ngroups;
  const int64_t r_end = cr0 + (cr1 - cr0) * (grp + 1) / g.ngroups;

  const int64_t c = static_cast<int64_t>(wig) * 32 + lane;
  const bool active = c < C;
  uint32_t xp[1][16];
  load_x_chunk<1>(p.x, 1, K, 32 * c, g.x_vec != 0, ASYM ? p.perm : nullptr, xp);
  int64_t scol = c;  // scale column of this lane's chunk
  bool mixed = false;
  if (ASYM && active) {
    const int64_t c0 = 32 * c;
    const int64_t last = (c0 + 31 < K) ? c0 + 31 : K - 1;
    scol = __ldg(p.g_idx + __ldg(p.perm + c0));
    mixed = scol != __ldg(p.g_idx + __ldg(p.perm + last));
  }
  const uint8_t *cptr = p.codes + 16 * c;
  const float *sptr = p.scales + scol;
  const int8_t *zptr = ASYM ? p.zeros + scol : nullptr;

  auto load_row = [&](int64_t r, RowData<ASYM> &d) {
    if (active && r < r_end) {
      d.c = ld_stream_v4(cptr + r * g.P);
      d.s = __ldg(sptr + r * g.SG);
      if (ASYM) d.z = static_cast<uint32_t>(static_cast<uint8_t>(__ldg(zptr + r * g.SG))) & 15u;
    } else {
      d.c = make_uint4(0u, 0u, 0u, 0u);
      d.s = 0.0f;
      d.z = 0u;
    }
  };

  RowData<ASYM> ring[kAhead];
#pragma unroll
  for (int i = 0; i < kAhead; ++i) load_row(r_begin + i, ring[i]);

  const int bar_id = 1 + grp;
  const int bar_threads = 32 * g.wg;
  int buf = 0;
  for (int64_t rb = r_begin; rb < r_end; rb += kGemvRows) {
    float acc[kGemvRows];
#pragma unroll
    for (int j = 0; j < kGemvRows; ++j) {
      const RowData<ASYM> d = ring[j % kAhead];
      load_row(rb + j + kAhead, ring[j % kAhead]);
      float v;
      if (!ASYM) {
        v = dot_chunk_ilp(d.c, xp[0], 0x43084308u, 0x43084308u) * d.s;
      } else if (!mixed) {
        v = dot_chunk_ilp(d.c, xp[0], 0x43004300u, (0x4300u | d.z) * 0x00010001u) * d.s;
      } else {
        // sorted columns of two groups share this chunk: per-column scale and zero
        v = 0.0f;
        const int64_t r = rb + j;
        if (active && r < r_end) {
          const uint32_t words[4] = {d.c.x, d.c.y, d.c.z, d.c.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int64_t col = 32 * c + 8 * t + e;
              if (col >= K) continue;
              const int64_t gg = __ldg(p.g_idx + __ldg(p.perm + col));
              const int u = static_cast<int>((words[t] >> (4 * e)) & 15u);
              const float w = __fmul_rn(static_cast<float>(u - p.zeros[r * g.SG + gg]), p.scales[r * g.SG + gg]);
              const uint32_t pair = xp[0][4 * t + (e & 3)];
              v = fmaf(__uint_as_float((e < 4 ? (pair & 0xFFFFu) : (pair >> 16)) << 16), w, v);
            }
          }
        }
      }
      acc[j] = v;
    }
    const float sum = reduce_rows8(acc, lane);
    if ((lane & 3) == 0) red[buf][warp][(lane >> 2) & 7] = sum;
    named_barrier_sync(bar_id, bar_threads);
    if (wig == 0 && lane < kGemvRows) {
      const int64_t n = rb + lane;
      if (n < r_end) {
        float v = 0.0f;
        for (int w = 0; w < g.wg; ++w) v += red[buf][grp * g.wg + w][lane];
        if (p.bias) v += __ldg(p.bias + n);
        if (p.y_dtype == W4_F32) {
          static_cast<float *>(p.y)[n] = v;
        } else {
          static_cast<__nv_bfloat16 *>(p.y)[n] = __float2bfloat16_rn(v);
        }
      }
    }
    buf ^= 1;  // the next block writes the other buffer; two barriers apart from this read
  }
}

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      count = n;
    else
      return 148;
  }
  return count;
}

bool make_geom(const LinearParams &p, RowsGeom *g, int *nw) {
  if (p.M != 1) return false;
  const int64_t K = p.K;
  const int64_t C = (K + 31) / 32;
  g->P = (K + 1) / 2;
  g->SG = p.asym ? p.n_groups : C;
  if (g->P % 16 != 0) return false;
  if (p.asym && p.perm == nullptr) return false;
  if (reinterpret_cast<uintptr_t>(p.codes) % 16 != 0) return false;
  const int64_t wg = (C + 31) / 32;
  if (wg > 28) return false;
  // 24 warps for rows of up to 4 warps (6 groups), else 28 (two groups of up to 14)
  *nw = wg <= 4 ? 24 : 28;
  g->wg = static_cast<int>(wg);
  g->ngroups = static_cast<int>(*nw / wg < 8 ? *nw / wg : 8);
  g->x_vec = (K % 8 == 0) && (reinterpret_cast<uintptr_t>(p.x) % 16 == 0);
  return true;
}

template <int NW, bool ASYM>
cudaError_t launch_typed(const LinearParams &p, const RowsGeom &g, cudaStream_t stream) {
  int64_t grid = (p.N + kGemvRows - 1) / kGemvRows;
  if (grid > sm_count()) grid = sm_count();
  gemv_rows_kernel<NW, ASYM><<<static_cast<unsigned>(grid), NW * 32, 0, stream>>>(p, g);
  return cudaGetLastError();
}

}  // namespace

bool gemv_rows_supports(const LinearParams &p) {
  RowsGeom g;
  int nw;
  return make_geom(p, &g, &nw);
}

cudaError_t launch_gemv_rows(const LinearParams &p, cudaStream_t stream) {
  RowsGeom g;
  int nw;
  if (!make_geom(p, &g, &nw)) return cudaErrorNotSupported;
  if (nw == 24) return p.asym ? launch_typed<24, true>(p, g, stream) : launch_typed<24, false>(p, g, stream);
  return p.asym ? launch_typed<28, true>(p, g, stream) : launch_typed<28, false>(p, g, stream);
}

}  // namespace w4i
