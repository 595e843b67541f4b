// Stage 2 of the Prox decode step (Prox §4.1 "Stage 2: exact sparse
// computation"; §4.3 fused output-sparse gate/up kernel and input-sparse
// down GEMV), and the dense SwiGLU baseline (Prox §2.1), which is the same
// phase with every channel kept.  Second phase of the fused per-token kernel
// (token.cu).
//
// Every CTA finds the token's exact top-k cut (select.cuh: key T and the tie
// cut) or applies the score threshold, lists the channels of its own range
// [F c / P, F (c + 1) / P) -- the channels it scored -- past it, ascending, at
// the range's start in a.sel_list and writes their count; once every CTA's
// count is in (a phase of the launch counter, token_args.cuh), CTA c takes
// the ranks [S c / P, S (c + 1) / P) of the whole selection (S channels,
// ascending), so every CTA streams the same number of channels (to one)
// whatever the mask looks like; a given list is split the same way by list
// position, and the dense baseline splits all channels.  Producer lanes
// stream, with 1-D bulk async copies (TMA engine) into a ring of slots, first
// the gate/up channel records of the CTA's channels (gate column then up
// column, d_model bf16 each: one copy per channel), then their W_down rows
// (two rows per slot).  The consumer warps
// take every ring item in order (so each mbarrier wait is for the phase right
// after one the waiting thread has already seen complete):
//   phase A: for each channel every warp of the owning group forms partial
//            dot products of its share of the column with the full x (x kept
//            in registers; fp32, packed f32x2 FMAs, warp-shuffle reduction)
//            and parks them in shared memory; after the last channel the
//            partials are summed in a fixed order into g = x . W_gate[:, j],
//            u = x . W_up[:, j] and s_j = act(g) u (the A3 ablation skips the
//            gate/up records and takes s_j = s~_j from Stage 1);
//   phase B: the warps accumulate y_part += s_j W_down[j, :] for the CTA's
//            channels, each thread owning 8-column groups of the output.
// The CTA's fp32 partial row goes to global memory as tagged words; the
// kernel adds the partial rows in a fixed order (token.cu).
#pragma once
#include "select.cuh"
#include "token_args.cuh"

namespace prox {
namespace s2 {

constexpr int NCW = kStage2Consumers;

// Layout of Stage 2's shared memory (bytes from the start): full and empty
// barriers [slots], s_val, s_idx [max_rec], s_pg, s_pu [max_rec][NCW], then
// the ring, 128-byte aligned (the selection's scratch and keys use the ring's
// bytes before the ring starts).
__host__ __device__ constexpr size_t ring_offset(int slots, int max_rec) {
  return ((size_t)slots * 16 + (size_t)max_rec * (8 + 8 * NCW) + 127) & ~(size_t)127;
}

// Selects the CTA's channels, streams them and writes the CTA's partial output
// row to a.ypart as tagged words (not in select_only mode; returns whether it
// did).  Every thread calls it.  MAXM =
// ceil(d_model / (8 * 32 * warps per group)): 8-element chunks per lane and
// column.
template <int MAXM>
__device__ bool run(const TokenArgs& a, unsigned char* smem, uint32_t tag, const uint32_t* hist,
                    const uint32_t* chist, const Phases& ph) {
  const int d = a.d, slots = a.slots;
  const uint32_t col_bytes = 2u * (uint32_t)d;     // one bf16 column / row
  const uint32_t slot_bytes = 2u * col_bytes;      // a gate/up record, or two W_down rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = gridDim.x, cta = blockIdx.x;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + slots;
  float* s_val = reinterpret_cast<float*>(empty + slots);        // [max_rec]
  int* s_idx = reinterpret_cast<int*>(s_val + a.max_rec);        // [max_rec]
  float* s_pg = reinterpret_cast<float*>(s_idx + a.max_rec);     // [max_rec][NCW]
  float* s_pu = s_pg + (size_t)a.max_rec * NCW;                  // [max_rec][NCW]
  unsigned char* ring = smem + ring_offset(slots, a.max_rec);

  // Consumer warps form NG groups of WPG; a group takes whole ring items, warp
  // wi of a group the elements [wi*qd, (wi+1)*qd) of each column / row
  // (qd = d / WPG), lane chunks e8 = m*32 + lane of 8 elements.
  const int NG = a.groups, WPG = NCW / NG, qd = d / WPG;
  const int grp = warp / WPG, wi = warp % WPG;
  auto elem = [&](int m) { return wi * qd + (m * 32 + lane) * 8; };
  auto elem_ok = [&](int m) { return (m * 32 + lane) * 8 < qd; };

  // The CTA's channels: ranks [r0, r0 + n) of the selection (ascending channel
  // order), of the list (list order) or of all channels (dense).
  int r0 = 0, n = 0;
  if (a.mode == kModeTopK || a.mode == kModeThreshold) {
    // this CTA's own channels (those it scored; their keys are in sc.own) past
    // the token's cut: the exact top-k cut, or the score threshold of Prox §4.1
    // (key >= bits(tau_s), every tie kept)
    SelectScratch& sc = *reinterpret_cast<SelectScratch*>(ring);
    TopkCut cut;
    if (a.mode == kModeTopK) {
      phase_wait(ph, 1);  // every CTA has counted its scores
      stamp(a.ts, 17);
      cut = select_cut(hist, chist, a.bucket, a.st64, a.F, a.k, sc, tag, a.err, a.ts);
      stamp(a.ts, 15);
    } else {
      cut.T = __float_as_uint(a.tau_s);
      cut.tie_cut = a.F;
    }
    const int c0 = (int)(((long long)a.F * cta) / P);
    const int m = (int)(((long long)a.F * (cta + 1)) / P) - c0;
    const bool sel = tid < m && selected(sc.own[tid], c0 + tid, cut);

    int own_n;
    const int pos = block_exclusive_scan(sel ? 1 : 0, sc.scan, &own_n);
    if (sel) st_tag(a.sel_list + c0 + pos, tag_word((uint32_t)(c0 + tid), tag));
    if (a.sel_mask && tid < m) a.sel_mask[c0 + tid] = sel ? 1 : 0;
    if (tid == 0) {
      st_tag(a.sel_cnt + cta, tag_word((uint32_t)own_n, tag));
      if (a.stats && !a.select_only) {
        if (cta == 0) atomicAdd(a.stats + 1, 1ull);
        atomicAdd(a.stats + 2, (unsigned long long)own_n);
      }
    }
    phase_arrive(ph);  // 2: counts written
    phase_wait(ph, 2);
    stamp(a.ts, 18);
    // every range's count
    int cnt = 0;
    if (tid < P) {
      unsigned long long w = ld_tag(a.sel_cnt + tid);
      const long long t0 = clock64();
      while (!tag_ok(w, tag) && wait_more(t0, a.err)) w = ld_tag(a.sel_cnt + tid);
      cnt = tag_ok(w, tag) ? (int)(uint32_t)w : 0;
    }
    int total;
    const int first = block_exclusive_scan(cnt, sc.scan, &total);
    if (tid < P) sc.own[tid] = (uint32_t)first;  // rank of range tid's first channel
    __syncthreads();
    // ranks [total c / P, total (c + 1) / P) of the selection, ascending:
    // rank q lives in the last range whose first rank is <= q
    r0 = (int)(((long long)total * cta) / P);
    n = (int)(((long long)total * (cta + 1)) / P) - r0;
    for (int i = tid; i < n; i += blockDim.x) {
      const int q = r0 + i;
      int lo = 0, hi = P - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int)sc.own[mid] <= q) lo = mid;
        else hi = mid - 1;
      }
      const unsigned long long* src = a.sel_list + (int)(((long long)a.F * lo) / P) + (q - (int)sc.own[lo]);
      unsigned long long w = ld_tag(src);
      const long long t0 = clock64();
      while (!tag_ok(w, tag) && wait_more(t0, a.err)) w = ld_tag(src);
      s_idx[i] = tag_ok(w, tag) ? (int)(uint32_t)w : 0;
    }
  } else {
    phase_arrive(ph);  // 2 (no counts to exchange)
    // list positions, or channels, [k c / P, k (c + 1) / P)
    const int k = a.mode == kModeDense ? a.F : a.k;
    r0 = (int)(((long long)k * cta) / P);
    n = (int)(((long long)k * (cta + 1)) / P) - r0;
    for (int i = tid; i < n; i += blockDim.x) {
      if (a.mode == kModeList) {
        int j = __ldcg(a.idx + r0 + i);
        if (j < 0 || j >= a.F) {
          atomicOr(a.err, PROX_DEVERR_MASK_INDEX);
          j = 0;
        }
        s_idx[i] = j;
      } else {
        s_idx[i] = r0 + i;
      }
    }
  }
  stamp(a.ts, 4);
  if (a.select_only) return false;

  // The ring and barriers take over bytes that the select (and Stage 1) wrote
  // through the generic proxy: order those writes before the bulk copies.
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW / NG);
    }
    fence_barrier_init();
  }
  __syncthreads();
  stamp(a.ts, 11);
  if (a.ts && tid == 0) a.ts[(size_t)cta * kPhaseStamps + 13] = (unsigned long long)n;

  // Ring items: channel records q < n (gate column | up column), then W_down
  // row pairs (rows 2p, 2p+1).  Group g takes records g, g+NG, ... and pairs
  // g, g+NG, ...; its items, records first, use the group's own SPG slots
  // [g*SPG, (g+1)*SPG) round robin, so every slot's waiter is one group that
  // takes its uses in order.  Producer lane g fills group g's slots.
  const int nB = (n + 1) >> 1;
  const int SPG = slots / NG;
  auto group_items = [&](int g, int cnt) { return cnt > g ? (cnt - g + NG - 1) / NG : 0; };
  unsigned long long* out_row = a.ypart + (size_t)cta * d;
  if (warp == NCW) {
    // ---------------- producer: one thread fills every group's slots ----------------
    // It polls the groups in turn with non-blocking tests, so a group that is
    // slow to free a slot never holds up the copies of another.
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int next[4] = {0, 0, 0, 0}, nA[4] = {0, 0, 0, 0}, tot[4] = {0, 0, 0, 0};
      int remaining = 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (g >= NG) continue;
        nA[g] = a.proxy_values ? 0 : group_items(g, n);
        tot[g] = nA[g] + group_items(g, nB);
        remaining += tot[g];
      }
      long long t_idle = clock64();
      bool pdead = false;
      while (remaining > 0 && !pdead) {
        bool progress = false;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          if (g >= NG) continue;
          const int li = next[g];
          if (li >= tot[g]) continue;
          const int slot = g * SPG + li % SPG, use = li / SPG;
          if (use > 0 && !mbar_test_wait(&empty[slot], (uint32_t)((use - 1) & 1))) continue;
          unsigned char* dst = ring + (size_t)slot * slot_bytes;
          if (li < nA[g]) {
            const int r = g + li * NG;
            mbar_arrive_expect_tx(&full[slot], slot_bytes);
            bulk_copy_g2s(dst, a.wgu + (size_t)s_idx[r] * 2 * (size_t)d, slot_bytes, &full[slot], pol);
          } else {
            const int r0 = 2 * (g + (li - nA[g]) * NG);
            const int nr = r0 + 1 < n ? 2 : 1;
            mbar_arrive_expect_tx(&full[slot], (uint32_t)nr * col_bytes);
            bulk_copy_g2s(dst, a.wd + (size_t)s_idx[r0] * (size_t)d, col_bytes, &full[slot], pol);
            if (nr == 2)
              bulk_copy_g2s(dst + col_bytes, a.wd + (size_t)s_idx[r0 + 1] * (size_t)d, col_bytes,
                            &full[slot], pol);
          }
          next[g] = li + 1;
          --remaining;
          progress = true;
        }
        if (progress) {
          t_idle = clock64();
        } else if (clock64() - t_idle > kWaitLimitCycles) {
          atomicOr(a.err, PROX_DEVERR_WAIT_TIMEOUT);
          pdead = true;
        }
      }
      // Every issued copy must land before this CTA's shared memory is reused:
      // wait for the last issued use of each slot (bounded).
      bool fdead = false;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (g >= NG) continue;
        for (int j = 0; j < SPG && j < next[g]; ++j) {
          const int last = j + ((next[g] - 1 - j) / SPG) * SPG;  // last li < next[g], li % SPG == j
          mbar_wait(&full[g * SPG + j], (uint32_t)((last / SPG) & 1), a.err, &fdead);
        }
      }
    }
  } else {
    // this thread's x elements, kept in registers
    float4 xr[MAXM][2];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = elem(m);
      xr[m][0] = elem_ok(m) ? __ldg(reinterpret_cast<const float4*>(a.x + e)) : make_float4(0, 0, 0, 0);
      xr[m][1] = elem_ok(m) ? __ldg(reinterpret_cast<const float4*>(a.x + e + 4)) : make_float4(0, 0, 0, 0);
    }
    bool cdead = false;
    // ---------------- phase A: gate/up partial dot products ----------------
    // The warp's share of an item goes into registers, the slot goes back to the
    // producer, then the FMAs.
    const int nA_g = a.proxy_values ? 0 : group_items(grp, n);
    for (int li = 0; li < nA_g; ++li) {
      const int r = grp + li * NG;
      const int slot = grp * SPG + li % SPG;
      mbar_wait(&full[slot], (uint32_t)((li / SPG) & 1), a.err, &cdead);
      const unsigned char* wg = ring + (size_t)slot * slot_bytes;
      const unsigned char* wu = wg + col_bytes;
      uint4 gv[MAXM], uv[MAXM];
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int e = elem(m);
        gv[m] = elem_ok(m) ? *reinterpret_cast<const uint4*>(wg + (size_t)e * 2) : make_uint4(0u, 0u, 0u, 0u);
        uv[m] = elem_ok(m) ? *reinterpret_cast<const uint4*>(wu + (size_t)e * 2) : make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot], 1);
      float2 ag0 = make_float2(0.f, 0.f), ag1 = ag0, au0 = ag0, au1 = ag0;
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const float4 xa = xr[m][0], xb = xr[m][1];
        ag0 = __ffma2_rn(bf16x2_to_f2(gv[m].x), make_float2(xa.x, xa.y), ag0);
        au0 = __ffma2_rn(bf16x2_to_f2(uv[m].x), make_float2(xa.x, xa.y), au0);
        ag1 = __ffma2_rn(bf16x2_to_f2(gv[m].y), make_float2(xa.z, xa.w), ag1);
        au1 = __ffma2_rn(bf16x2_to_f2(uv[m].y), make_float2(xa.z, xa.w), au1);
        ag0 = __ffma2_rn(bf16x2_to_f2(gv[m].z), make_float2(xb.x, xb.y), ag0);
        au0 = __ffma2_rn(bf16x2_to_f2(uv[m].z), make_float2(xb.x, xb.y), au0);
        ag1 = __ffma2_rn(bf16x2_to_f2(gv[m].w), make_float2(xb.z, xb.w), ag1);
        au1 = __ffma2_rn(bf16x2_to_f2(uv[m].w), make_float2(xb.z, xb.w), au1);
      }
      float g = (ag0.x + ag0.y) + (ag1.x + ag1.y);
      float u = (au0.x + au0.y) + (au1.x + au1.y);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        u += __shfl_xor_sync(0xffffffffu, u, o);
      }
      if (lane == 0) {
        s_pg[r * NCW + wi] = g;
        s_pu[r * NCW + wi] = u;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    for (int r = tid; r < n; r += NCW * 32) {
      float sv;
      if (a.proxy_values) {
        unsigned long long w = ld_tag(a.st64 + s_idx[r]);
        const long long t0 = clock64();
        while (!tag_ok(w, tag) && wait_more(t0, a.err)) w = ld_tag(a.st64 + s_idx[r]);
        sv = __uint_as_float((uint32_t)w);
      } else {
        float g = 0.f, u = 0.f;
        for (int w = 0; w < WPG; ++w) {
          g += s_pg[r * NCW + w];
          u += s_pu[r * NCW + w];
        }
        sv = act_f32(g, a.act) * u;
      }
      s_val[r] = sv;
      if (a.s_sp) a.s_sp[r0 + r] = sv;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    stamp(a.ts, 12);

    // ---------------- phase B: y_part = sum_t s_t W_down[j_t, :] ----------------
    // The group's row pairs; warp wi accumulates its columns [wi*qd, (wi+1)*qd).
    float2 acc[MAXM * 4];
#pragma unroll
    for (int i = 0; i < MAXM * 4; ++i) acc[i] = make_float2(0.f, 0.f);
    const int nB_g = group_items(grp, nB);
    for (int lb = 0; lb < nB_g; ++lb) {
      const int li = nA_g + lb;
      const int p = grp + lb * NG;  // row pair
      const int slot = grp * SPG + li % SPG;
      mbar_wait(&full[slot], (uint32_t)((li / SPG) & 1), a.err, &cdead);
      const unsigned char* w = ring + (size_t)slot * slot_bytes;
      const bool two = 2 * p + 1 < n;
      uint4 wv[2][MAXM];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          const int e = elem(m);
          wv[h][m] = (elem_ok(m) && (h == 0 || two))
                         ? *reinterpret_cast<const uint4*>(w + h * col_bytes + (size_t)e * 2)
                         : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot], 1);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float sv = (h == 0 || two) ? s_val[2 * p + h] : 0.f;
        const float2 s2 = make_float2(sv, sv);
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          const uint4 w4 = wv[h][m];
          acc[4 * m + 0] = __ffma2_rn(bf16x2_to_f2(w4.x), s2, acc[4 * m + 0]);
          acc[4 * m + 1] = __ffma2_rn(bf16x2_to_f2(w4.y), s2, acc[4 * m + 1]);
          acc[4 * m + 2] = __ffma2_rn(bf16x2_to_f2(w4.z), s2, acc[4 * m + 2]);
          acc[4 * m + 3] = __ffma2_rn(bf16x2_to_f2(w4.w), s2, acc[4 * m + 3]);
        }
      }
    }
    // The groups' partial rows are added in group order (deterministic).  Every
    // copy has landed (each item was waited for), so the ring holds them.
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    float* s_y = reinterpret_cast<float*>(ring);  // [NG][d]
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      if (elem_ok(m)) {
        float* dst = s_y + (size_t)grp * d + elem(m);
        *reinterpret_cast<float4*>(dst) =
            make_float4(acc[4 * m].x, acc[4 * m].y, acc[4 * m + 1].x, acc[4 * m + 1].y);
        *reinterpret_cast<float4*>(dst + 4) =
            make_float4(acc[4 * m + 2].x, acc[4 * m + 2].y, acc[4 * m + 3].x, acc[4 * m + 3].y);
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    // one 16-byte tagged pair per lane and store: each warp store covers
    // whole sectors
    for (int e = tid * 2; e < d; e += NCW * 32 * 2) {
      float2 v = *reinterpret_cast<const float2*>(s_y + e);
      for (int g = 1; g < NG; ++g) {
        const float2 t = *reinterpret_cast<const float2*>(s_y + (size_t)g * d + e);
        v.x += t.x;
        v.y += t.y;
      }
      st_tag2(out_row + e, tag_word(__float_as_uint(v.x), tag), tag_word(__float_as_uint(v.y), tag));
    }
  }
  return true;
}

}  // namespace s2
}  // namespace prox
