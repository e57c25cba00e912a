// act_quant.cu -- online NVFP4 quantization of activations: a dynamic global
// scale per token and the plain-MSE scale sweep, fused in one kernel.
//
// ScaleSweep summary, sec. 1-3 and "Experimental Results" (the W+A settings):
// activations are NVFP4 as well, quantized with the MSE objective and the
// [-3, +7] window.  Where the page is silent the reading is: the FP32 global
// scale is dynamic, one per token, S_t = fl32(amax_t / fl32(Q * 6)) by the
// same formula as for a weight tensor, and each token row is then swept as a
// one-row matrix (every group decided exactly as in scale_sweep.cu, h == 1).
//
// Work layout: a team of TW warps (TW = 1, 2 or 4 of the CTA's four) owns one
// token row at a time over a one-wave grid.  Each team starts with the row of
// its own index; with at least four rows per team it takes every further row
// from a leased counter (row_counters.cuh) as it finishes one, otherwise it
// strides by the number of teams.
//   Pass 1 reads the row with 16-byte loads and takes the max of the
//   sign-cleared bf16 bit patterns: a warp reduction, then for TW > 1 an
//   exchange through shared memory under a named barrier of the team.
//   Pass 2 sweeps the row's groups.  Team lane l takes groups l, l + 32 TW, ...;
//   the next group's 32 bytes are copied into shared memory with cp.async
//   while the current one is scored.  The row was read a moment before under
//   an evict-last L2 policy, so those copies hit L2 and DRAM sees each byte
//   once.
#include <type_traits>

#include "nvfp4hs.h"
#include "nvfp4_kernels.cuh"
#include "row_counters.cuh"
#include "sweep_core.cuh"

namespace nvfp4 {

namespace {

// Named barrier of one team (ids 1 and 2 as immediates, so the kernel
// reserves only the barriers it uses; id 0 is __syncthreads).
template <int kThreads>
__device__ __forceinline__ void team_barrier(int team) {
  if (team == 0)
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
  else
    asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
}

// CTAs per SM the compile-time 11-candidate form is built for (it needs the
// fewest registers; more resident warps hide more latency).
constexpr int kActCtas11 = 7;

// L2 eviction priorities for the row's two reads.  Pass 1 marks the row
// evict-last so that it is still in L2 when pass 2 reads it back; pass 2
// marks it evict-first once used.  Without them about 60% of the rows were
// read from DRAM a second time.
__device__ __forceinline__ uint64_t l2_policy(bool keep) {
  uint64_t pol;
  if (keep)
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ld_v4_policy(const void* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ void cp_async16_policy(void* smem, const void* gmem, uint64_t pol) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem),
               "l"(pol)
               : "memory");
}

template <int TW, int kK>
__global__ void __launch_bounds__(kCta, kK == 11 ? kActCtas11 : 5)
act_quant_kernel(const uint16_t* __restrict__ A, int64_t tokens, int64_t G, int64_t lda,
                 float q_max, int lo, int hi, float* __restrict__ S_out,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                 int8_t* __restrict__ offs, int* __restrict__ status,
                 unsigned int* __restrict__ slot) {
  __shared__ SweepSmem<16> sm;
  __shared__ uint32_t red[2][kCta / 32];  // per-warp row maxima, by row parity
  __shared__ uint32_t nxt[2][kCta / 32];  // next row of each team, by row parity
  fill_candidate_table(sm.tab);
  __syncthreads();

  constexpr int kTeams = (kCta / 32) / TW;
  constexpr int kTeamThreads = 32 * TW;
  const int lane = threadIdx.x;
  const int warp = lane >> 5;
  const int team = warp / TW;
  const int tl = lane - team * kTeamThreads;  // position in the team
  const int64_t nteams = static_cast<int64_t>(gridDim.x) * kTeams;
  const int64_t nvec = G * 2;                  // 16-byte vectors per row
  const int64_t half_in = G * 8;
  const float q6 = __fmul_rn(q_max, 6.0f);
  const int K = hi - lo + 1;
  auto& wbuf = sm.wbuf;

  f32x2_t ones[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ones[i] = f2_pack(1.0f, 1.0f);

  const uint64_t keep = l2_policy(true), drop = l2_policy(false);
  int parity = 0, buf = 0;
  int64_t t = static_cast<int64_t>(blockIdx.x) * kTeams + team;
  while (t < tokens) {
    const uint16_t* row = A + t * lda;
    // the next row, taken now and used once this one is done
    uint32_t grab = 0;
    if (slot != nullptr && tl == 0) grab = atomicAdd(slot, 1u);

    // ---- pass 1: the row's absmax as a bf16 bit pattern
    uint32_t m2 = 0;
    int64_t v = tl;
    for (; v + 3 * kTeamThreads < nvec; v += 4 * kTeamThreads) {
      uint4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = ld_v4_policy(row + (v + u * kTeamThreads) * 8, keep);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        m2 = __vmaxu2(__vmaxu2(m2, x[u].x & 0x7FFF7FFFu),
                      __vmaxu2(__vmaxu2(x[u].y & 0x7FFF7FFFu, x[u].z & 0x7FFF7FFFu),
                               x[u].w & 0x7FFF7FFFu));
    }
    for (; v < nvec; v += kTeamThreads) {
      const uint4 x = ld_v4_policy(row + v * 8, keep);
      m2 = __vmaxu2(__vmaxu2(m2, x.x & 0x7FFF7FFFu),
                    __vmaxu2(__vmaxu2(x.y & 0x7FFF7FFFu, x.z & 0x7FFF7FFFu), x.w & 0x7FFF7FFFu));
    }
    uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    // the next row's index waits in shared memory (read once this row is
    // done; the slot of this parity is not written again before the team
    // has passed the next row's barrier)
    if (tl == 0) nxt[parity][team] = grab;
    if constexpr (TW > 1) {
      if ((lane & 31) == 0) red[parity][warp] = mb;
      team_barrier<kTeamThreads>(team);
#pragma unroll
      for (int i = 0; i < TW; ++i) mb = max(mb, red[parity][team * TW + i]);
    } else {
      __syncwarp();
    }

    // S_t = fl32(amax / fl32(Q * 6)); Inf or NaN in the row (a pattern at or
    // above 0x7F80) gives S_t = NaN, a zero row and the status word
    const bool nonfinite = mb >= 0x7F80u;
    const float S = nonfinite ? __uint_as_float(0x7FC00000u)
                              : __fdiv_rn(__uint_as_float(mb << 16), q6);
    if (tl == 0) {
      S_out[t] = S;
      if (nonfinite && status) *status = NVFP4_ERR_NONFINITE;
    }
    uint8_t* crow = codes + t * half_in;
    uint8_t* srow = scales + t * G;
    int8_t* orow = offs ? offs + t * G : nullptr;
    if (nonfinite) {
      for (int64_t g = tl; g < G; g += kTeamThreads) {
        *reinterpret_cast<uint2*>(crow + g * 8) = make_uint2(0u, 0u);
        srow[g] = 0;
        if (orow) orow[g] = 0;
      }
      t = slot != nullptr ? nteams + nxt[parity][team] : t + nteams;
      parity ^= 1;
      continue;
    }

    // ---- pass 2: sweep the row's groups with this row's S
    const ScaleConsts sc = scale_consts(S);
    auto issue = [&](int64_t gg, int b) {
      const uint16_t* src = row + gg * 16;
      cp_async16_policy(&wbuf[b][0][lane], src, drop);
      cp_async16_policy(&wbuf[b][1][lane], src + 8, drop);
    };
    if (tl < G) issue(tl, buf);
    cp_async_commit();
    for (int64_t g = tl; g < G; g += kTeamThreads) {
      const unsigned amask = __activemask();
      if (g + kTeamThreads < G) issue(g + kTeamThreads, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
      const int cur = buf;
      buf ^= 1;
      sweep_group<false, false, 16, kK>(sm, amask, cur, ones, 1.0f, 16.0f, nullptr, g, sc, lo, K,
                                    [&](uint2 c, uint8_t s, int8_t o) {
                                      *reinterpret_cast<uint2*>(crow + g * 8) = c;
                                      srow[g] = s;
                                      if (orow) orow[g] = o;
                                    });
    }
    cp_async_wait<0>();
    t = slot != nullptr ? nteams + nxt[parity][team] : t + nteams;
    parity ^= 1;
  }
  if (slot != nullptr) finish_slot(slot, 1);
}

}  // namespace

// Resident CTAs per SM of the instantiation launched for a team size and
// window (the 11-candidate form holds more CTAs than the general one).
int act_quant_resident_ctas(int tw, bool k11) {
  static const int n[3][2] = {
      {resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<1, 0>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<1, 11>), kCta)},
      {resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<2, 0>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<2, 11>), kCta)},
      {resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<4, 0>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&act_quant_kernel<4, 11>), kCta)}};
  return n[tw == 1 ? 0 : (tw == 2 ? 1 : 2)][k11 ? 1 : 0];
}

int act_quant_team_warps(int64_t tokens, int64_t in, int num_sms, bool k11) {
  // cost of a team size: rounds of rows per team x groups per lane per row,
  // times the team's own overhead (the exchange and barrier of each row, and
  // fewer rows in flight per SM), measured on B200 as about 5% for two warps
  // and 15% for four at equal parallelism.  The smallest cost wins: a large
  // batch gets one warp per row, a small one spreads each row over four.
  const int64_t G = in / 16;
  const double overhead[3] = {1.0, 1.05, 1.15};
  int best_tw = 1;
  double best = -1.0;
  for (int i = 0, tw = 1; tw <= 4; ++i, tw *= 2) {
    const int64_t wave_warps =
        static_cast<int64_t>(num_sms) * act_quant_resident_ctas(tw, k11) * (kCta / 32);
    const int64_t teams = wave_warps / tw;
    const int64_t rounds = (tokens + teams - 1) / teams;
    const int64_t per_row = (G + 32 * tw - 1) / (32 * tw);
    const double cost = static_cast<double>(rounds * (per_row > 0 ? per_row : 1)) * overhead[i];
    if (best < 0.0 || cost < best) { best = cost; best_tw = tw; }
  }
  return best_tw;
}

cudaError_t launch_quantize_activations(const uint16_t* A, int64_t tokens, int64_t in,
                                        int64_t lda, float q_max, int lo, int hi, float* S,
                                        uint8_t* codes, uint8_t* scales, int8_t* offs,
                                        int* status, int num_sms, cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  const bool k11 = hi - lo + 1 == 11;
  const int tw = act_quant_team_warps(tokens, in, num_sms, k11);
  const int64_t teams_per_cta = (kCta / 32) / tw;
  int64_t blocks = (tokens + teams_per_cta - 1) / teams_per_cta;
  const int64_t wave = static_cast<int64_t>(num_sms) * act_quant_resident_ctas(tw, k11);
  if (blocks > wave) blocks = wave;
  const int64_t G = in / 16;
  const unsigned nb = static_cast<unsigned>(blocks);
  // rows from a counter once every team would take four rows or more
  CounterLease lease(stream, tokens >= 4 * blocks * teams_per_cta && tokens < (int64_t{1} << 31));
  unsigned int* slot = lease.slot();
  // the page's [-3, +7] window (11 candidates) gets a compile-time count
  auto launch = [&](auto tw_c, auto kk) {
    act_quant_kernel<decltype(tw_c)::value, decltype(kk)::value><<<nb, kCta, 0, stream>>>(
        A, tokens, G, lda, q_max, lo, hi, S, codes, scales, offs, status, slot);
  };
  using T11 = std::integral_constant<int, 11>;
  using T0 = std::integral_constant<int, 0>;
  if (tw == 1) {
    if (k11) launch(std::integral_constant<int, 1>{}, T11{}); else launch(std::integral_constant<int, 1>{}, T0{});
  } else if (tw == 2) {
    if (k11) launch(std::integral_constant<int, 2>{}, T11{}); else launch(std::integral_constant<int, 2>{}, T0{});
  } else {
    if (k11) launch(std::integral_constant<int, 4>{}, T11{}); else launch(std::integral_constant<int, 4>{}, T0{});
  }
  return lease.commit(cudaGetLastError());
}

}  // namespace nvfp4
