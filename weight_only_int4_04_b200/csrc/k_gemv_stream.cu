// Streaming decode GEMV, the M = 1 path:
//   y[m][n] = sum_k x[m][k] * w[n][k] + b[n]
//
// The packed rows of a weight are contiguous in HBM (codes [N, P] then scales [N, G]), so a
// block of rows is ONE contiguous byte range of each array. Each CTA (one per SM) owns a
// balanced contiguous range of rows and streams it through a ring of shared-memory slots of
// 8 rows each:
//   * a producer thread issues one cp.async.bulk per array per slot (the bulk-copy engine
//     keeps the whole ring -- up to ~200 KB per SM -- in flight, far above what HBM needs
//     to run at full rate), completing on the slot's "full" mbarrier;
//   * consumer warps own 32-column chunks (lane = chunk = one scale group = 16 code bytes),
//     hold their activation chunk in registers for the whole kernel, and read the codes of
//     each row from shared memory (512 contiguous bytes per warp instruction, conflict
//     free). Nibble pairs become exact bf16x2 integers (one LOP3 each: the nibble drops into
//     the mantissa of 128.0, whose ulp is 1; one exact bf16x2 FMA removes the offset) and
//     meet the activations in sm_100 mixed-precision FMAs (bf16 x bf16 + fp32, full rate,
//     the product is exact) in four independent chains; the group scale multiplies the fp32
//     partial. The warps that together cover all chunks of a row form a group; with
//     short rows several groups split the slots round-robin;
//   * per slot, the group reduces 8 rows across lanes (transposing butterfly) and across
//     its warps (shared memory, fixed order: deterministic), writes y and frees the slot.
// Asymmetric act-order codes (sorted by w4_asym_prepare) take the same path with per-chunk
// zero points and x gathered through perm once per CTA.
#include "w4_dot.cuh"
#include "w4_sync.cuh"

namespace w4i {

namespace {

constexpr int kMaxConsumerWarps = 28;
constexpr int kMaxSlots = 16;
constexpr int kMaxCpl = 1;  // chunks per lane (K <= 16384)
constexpr int kSmemBudget = 216 * 1024;

struct StreamGeom {
  int nw;           // consumer warps of the launch (24 or 28)
  int64_t P;        // code bytes per row
  int64_t SG;       // scale (and zero) columns per row
  int slot_bytes;   // 8 rows of codes + scales (+ zeros)
  int scales_off;   // offsets inside a slot
  int zeros_off;
  int nslots;
  int wg;           // warps per group: ceil(C / 32), at most 16
  int ngroups;      // 16 / wg
  int cpl;          // chunks per lane
  int spg;          // slots per group (each group walks its own ring)
  int x_vec;        // 16-byte activation loads allowed
};

// Shared-memory tail after the slots: reduction buffers, barriers and the abort flag.
constexpr int kRedBytes = 2 * kMaxConsumerWarps * kGemvRows * 2 * 4;
constexpr int kTailBytes = kRedBytes + 2 * kMaxSlots * 8 + 16;

template <int MT, bool ASYM, int CPL, int NW>
__global__ void __launch_bounds__(32 * (NW + 1), 1)
    gemv_stream_kernel(const LinearParams p, const StreamGeom g, int32_t *err) {
  extern __shared__ __align__(128) uint8_t smem[];
  float *red = reinterpret_cast<float *>(smem + static_cast<size_t>(g.nslots) * g.slot_bytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + kRedBytes);
  uint64_t *empty = full + kMaxSlots;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kMaxSlots);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = p.N, K = p.K, M = p.M;
  const int64_t C = (K + 31) / 32;
  const int64_t row_begin = static_cast<int64_t>(blockIdx.x) * N / gridDim.x;
  const int64_t row_end = static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x;
  const int nstages = static_cast<int>((row_end - row_begin + kGemvRows - 1) / kGemvRows);

  if (threadIdx.x == 0) {
    for (int i = 0; i < g.nslots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---- producer: one thread streams the CTA's rows through the slot ring ----
    if (lane == 0) {
      for (int s = 0; s < nstages; ++s) {
        // stage s belongs to group s % ngroups, which walks its own ring of spg slots
        const int kq = s / g.ngroups;
        const int slot = (s % g.ngroups) * g.spg + kq % g.spg;
        const uint32_t ph = static_cast<uint32_t>(kq / g.spg) & 1u;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag, err)) break;
        const int64_t r0 = row_begin + static_cast<int64_t>(s) * kGemvRows;
        const int64_t nr = (row_end - r0) < kGemvRows ? (row_end - r0) : kGemvRows;
        uint8_t *base = smem + static_cast<size_t>(slot) * g.slot_bytes;
        const uint32_t cb = static_cast<uint32_t>(nr * g.P);
        const uint32_t sb = static_cast<uint32_t>(nr * g.SG * 4);
        const uint32_t zb = ASYM ? static_cast<uint32_t>(nr * g.SG) : 0u;
        mbar_arrive_expect_tx(&full[slot], cb + sb + zb);
        bulk_copy_g2s(base, p.codes + r0 * g.P, cb, &full[slot]);
        bulk_copy_g2s(base + g.scales_off, p.scales + r0 * g.SG, sb, &full[slot]);
        if (ASYM) bulk_copy_g2s(base + g.zeros_off, p.zeros + r0 * g.SG, zb, &full[slot]);
      }
    }
    return;
  }

  // ---- consumers ----
  const int cw = warp - 1;
  const int grp = cw / g.wg, wig = cw % g.wg;
  if (grp >= g.ngroups) return;

  uint32_t xp[CPL][MT][16];
  int64_t chunk[CPL];
  int64_t cgroup[CPL];  // asym: scale column of the chunk
  bool mixed[CPL];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    chunk[j] = static_cast<int64_t>(wig) * 32 + lane + static_cast<int64_t>(j) * g.wg * 32;
    load_x_chunk<MT>(p.x, M, K, 32 * chunk[j], g.x_vec != 0, ASYM ? p.perm : nullptr, xp[j]);
    cgroup[j] = 0;
    mixed[j] = false;
    if (ASYM && chunk[j] < C) {
      const int64_t c0 = 32 * chunk[j];
      const int64_t last = (c0 + 31 < K) ? c0 + 31 : K - 1;
      cgroup[j] = __ldg(p.g_idx + __ldg(p.perm + c0));
      mixed[j] = cgroup[j] != __ldg(p.g_idx + __ldg(p.perm + last));
    }
  }

  const int bar_id = 1 + grp;
  const int bar_threads = 32 * g.wg;
  int buf = 0;
  for (int s = grp; s < nstages; s += g.ngroups) {
    const int kq = s / g.ngroups;
    const int slot = grp * g.spg + kq % g.spg;
    const uint32_t ph = static_cast<uint32_t>(kq / g.spg) & 1u;
    mbar_wait(&full[slot], ph, abort_flag, err);  // on failure: finish the pass on stale data
    const int64_t r0 = row_begin + static_cast<int64_t>(s) * kGemvRows;
    const int nr = static_cast<int>((row_end - r0) < kGemvRows ? (row_end - r0) : kGemvRows);
    const uint8_t *sc = smem + static_cast<size_t>(slot) * g.slot_bytes;
    const float *ss = reinterpret_cast<const float *>(sc + g.scales_off);
    const int8_t *sz = reinterpret_cast<const int8_t *>(sc + g.zeros_off);

    float acc[kGemvRows][MT];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) {
      if (r < nr) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          if (chunk[j] < C) {
            const uint4 cw4 = *reinterpret_cast<const uint4 *>(sc + r * g.P + 16 * chunk[j]);
            if (!ASYM) {
              const float scale = ss[r * g.SG + chunk[j]];
#pragma unroll
              for (int m = 0; m < MT; ++m)
                acc[r][m] = fmaf(dot_chunk_ilp(cw4, xp[j][m], 0x43084308u, 0x43084308u), scale, acc[r][m]);
            } else if (!mixed[j]) {
              const float scale = ss[r * g.SG + cgroup[j]];
              const uint32_t z = static_cast<uint32_t>(static_cast<uint8_t>(sz[r * g.SG + cgroup[j]])) & 15u;
#pragma unroll
              for (int m = 0; m < MT; ++m)
                acc[r][m] = fmaf(dot_chunk_ilp(cw4, xp[j][m], 0x43004300u, (0x4300u | z) * 0x00010001u), scale,
                                 acc[r][m]);
            } else {
              // sorted columns of two groups share this chunk: per-column scale and zero
              const uint32_t words[4] = {cw4.x, cw4.y, cw4.z, cw4.w};
#pragma unroll
              for (int t = 0; t < 4; ++t) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int64_t col = 32 * chunk[j] + 8 * t + e;
                  if (col >= K) continue;
                  const int64_t gg = __ldg(p.g_idx + __ldg(p.perm + col));
                  const int u = static_cast<int>((words[t] >> (4 * e)) & 15u);
                  const float w = __fmul_rn(static_cast<float>(u - sz[r * g.SG + gg]), ss[r * g.SG + gg]);
#pragma unroll
                  for (int m = 0; m < MT; ++m) {
                    const uint32_t pair = xp[j][m][4 * t + (e & 3)];
                    acc[r][m] = fmaf(__uint_as_float((e < 4 ? (pair & 0xFFFFu) : (pair >> 16)) << 16), w,
                                     acc[r][m]);
                  }
                }
              }
            }
          }
        }
      }
    }

    float *rb = red + buf * (kMaxConsumerWarps * kGemvRows * 2);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v[kGemvRows];
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r) v[r] = acc[r][m];
      const float sum = reduce_rows8(v, lane);
      if ((lane & 3) == 0) rb[(cw * kGemvRows + ((lane >> 2) & 7)) * 2 + m] = sum;
    }
    named_barrier_sync(bar_id, bar_threads);
    if (wig == 0) {
      if (lane < kGemvRows * MT) {
        const int r = lane / MT, m = lane % MT;
        if (r < nr && m < M) {
          float v = 0.0f;
          for (int w = 0; w < g.wg; ++w) v += rb[((grp * g.wg + w) * kGemvRows + r) * 2 + m];
          const int64_t n = r0 + r;
          if (p.bias) v += __ldg(p.bias + n);
          if (p.y_dtype == W4_F32) {
            static_cast<float *>(p.y)[m * N + n] = v;
          } else {
            static_cast<__nv_bfloat16 *>(p.y)[m * N + n] = __float2bfloat16_rn(v);
          }
        }
      }
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    buf ^= 1;
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

bool make_geom(const LinearParams &p, StreamGeom *g) {
  if (p.M != 1) return false;
  const int64_t K = p.K;
  const int64_t C = (K + 31) / 32;
  g->P = (K + 1) / 2;
  g->SG = p.asym ? p.n_groups : C;
  if (g->P % 16 != 0) return false;
  if (p.asym && (p.perm == nullptr || g->SG % 16 != 0)) return false;
  if (!p.asym && g->SG % 4 != 0) return false;
  const uintptr_t align = reinterpret_cast<uintptr_t>(p.codes) | reinterpret_cast<uintptr_t>(p.scales) |
                          (p.asym ? reinterpret_cast<uintptr_t>(p.zeros) : 0);
  if (align % 16 != 0) return false;
  const int64_t wg0 = (C + 31) / 32;
  if (wg0 > kMaxConsumerWarps) return false;
  // 24 consumer warps when rows need at most 4 warps, else 28 (two groups of up to 14)
  const int nw = wg0 <= 4 ? 24 : 28;
  const int64_t wg = wg0;
  const int64_t cpl = (C + wg * 32 - 1) / (wg * 32);
  if (cpl > kMaxCpl) return false;
  const int64_t codes_b = kGemvRows * g->P;
  const int64_t scales_b = kGemvRows * g->SG * 4;
  const int64_t zeros_b = p.asym ? kGemvRows * g->SG : 0;
  const int64_t slot = codes_b + scales_b + ((zeros_b + 127) / 128) * 128;
  const int64_t nslots = (kSmemBudget - kTailBytes) / slot;
  if (nslots < 2) return false;
  g->slot_bytes = static_cast<int>(slot);
  g->scales_off = static_cast<int>(codes_b);
  g->zeros_off = static_cast<int>(codes_b + scales_b);
  const int64_t ns = nslots < kMaxSlots ? nslots : kMaxSlots;
  int64_t ngroups = nw / wg < 8 ? nw / wg : 8;  // named barriers 1..8
  if (ngroups > ns / 2) ngroups = ns / 2;
  g->wg = static_cast<int>(wg);
  g->ngroups = static_cast<int>(ngroups);
  g->spg = static_cast<int>(ns / ngroups);
  g->nslots = static_cast<int>(ngroups * g->spg);
  g->cpl = static_cast<int>(cpl);
  g->x_vec = (K % 8 == 0) && (reinterpret_cast<uintptr_t>(p.x) % 16 == 0);
  g->nw = nw;
  return true;
}

template <int MT, bool ASYM, int CPL, int NW>
cudaError_t launch_typed(const LinearParams &p, const StreamGeom &g, int32_t *err, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(g.nslots) * g.slot_bytes + kTailBytes;
  auto kern = gemv_stream_kernel<MT, ASYM, CPL, NW>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int64_t grid = (p.N + kGemvRows - 1) / kGemvRows;
  if (grid > sm_count()) grid = sm_count();
  kern<<<static_cast<unsigned>(grid), 32 * (NW + 1), smem, stream>>>(p, g, err);
  return cudaGetLastError();
}

}  // namespace

bool gemv_stream_supports(const LinearParams &p) {
  StreamGeom g;
  return make_geom(p, &g);
}

cudaError_t launch_gemv_stream(const LinearParams &p, int32_t *err, cudaStream_t stream) {
  StreamGeom g;
  if (!make_geom(p, &g)) return cudaErrorNotSupported;
  if (g.nw == 24)
    return p.asym ? launch_typed<1, true, 1, 24>(p, g, err, stream) : launch_typed<1, false, 1, 24>(p, g, err, stream);
  return p.asym ? launch_typed<1, true, 1, 28>(p, g, err, stream) : launch_typed<1, false, 1, 28>(p, g, err, stream);
}

}  // namespace w4i
