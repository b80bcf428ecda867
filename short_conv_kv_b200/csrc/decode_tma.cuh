// Fused ShortConv K/V decode step, streaming version (sm_100a): one new
// token per sequence.
//
// Persistent CTAs (x) over the batch, channel slices of <= 256 groups of 8
// channels (y).  CTA b handles sequences b, b + ctas, b + 2*ctas, ... (at
// most kDecMaxSeqs).  In a prologue its threads read every such sequence's
// state index and slot into shared memory, so the copies need no further
// index round trips.
//
// One ring stage per sequence holds W rows of the CTA's slice: the W-1 old
// state rows (oldest first) and the new K/V row, brought in by bulk
// asynchronous copies (thread 0 issues them, the first sequence's alone and
// the rest once it has landed; completion counted in bytes on the stage's
// "full" barrier).  Once a stage has landed:
//   - the new state is exactly stage rows 1..W-1 (old rows 1..W-2, then the
//     new row), so thread 0 writes it back with bulk shared->global copies
//     over the rows just read -- the state update never passes through
//     registers (with a ring-buffer state only the new row is written, into
//     the row of the oldest position);
//   - every thread convolves its 8 channels over the W rows, reduces the
//     head's sum of squares by xor shuffles, and stores its 16 bytes of the
//     normalised bf16 row into the cache slot.
// Thread 0 waits until its write-back has finished reading the stage before
// the stage is released for the next sequence.
#pragma once
#include "common.cuh"
#include "tma.cuh"

namespace sconv {

constexpr int kDecMaxSeqs = 64;  // sequences per CTA (prologue index tables)
#ifndef SCONV_DECODE_EARLY_STAGES
#define SCONV_DECODE_EARLY_STAGES 1  // early state fetch: sequences requested before the wait
#endif

struct DecGeom {
  int slice;      // channel groups per full slice (min(NG, 256))
  int stages;     // ring depth (sequences in flight per CTA)
  int ctas;       // CTAs along the batch
  int withhold_first;  // testing: the first sequence's copies are never made
  int smem_ring;  // bytes of the ring
  int state_early;  // first sequence's state rows requested before the dependency wait
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store has finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// CTAs per SM by register need: four (<= 64 registers) for W <= 4, three
// for W = 5, two beyond.
template <int W>
__host__ __device__ constexpr int decode_ctas_per_sm() { return W <= 4 ? 4 : (W == 5 ? 3 : 2); }
inline int decode_ctas_per_sm(int W) { return W <= 4 ? 4 : (W == 5 ? 3 : 2); }

template <int W, int D, bool MX, bool LV>
__global__ void __launch_bounds__(256, decode_ctas_per_sm<W>())
    decode_tma_kernel(const StepParams P, const DecGeom Gm) {
  extern __shared__ __align__(128) unsigned char smem[];
  // layout variants only in the LV instances (compile-time defaults elsewhere)
  const int64_t gamma_hs = LV ? P.gamma_hs : 0;
  const int64_t* const state_pos = LV ? P.state_pos : nullptr;
  constexpr int G = D / 8;
  const int B = P.num_seqs;
  const int NS = Gm.stages;

  const int half = P.NG >> 1;
  const int g0 = blockIdx.y * Gm.slice;
  const int cs = min(Gm.slice, P.NG - g0);
  const int ncw = (cs + 31) >> 5;
  const int kn = max(0, min(g0 + cs, half) - g0);
  const int vg0 = max(g0, half);
  const int vn = max(0, g0 + cs - vg0);
  const int row_bytes = cs * 16;
  const int stage_bytes = W * row_bytes;
  const bool full_slice = (cs == P.NG);
  const int64_t srow = 2 * static_cast<int64_t>(P.C);

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Gm.smem_ring);
  uint64_t* empty = full + NS;
  long long* s_off = reinterpret_cast<long long*>(empty + NS);  // cache row offset or -1
  long long* s_si = s_off + kDecMaxSeqs;                        // state row, -1 = skip
  // ring-buffer state: row of the window's oldest position (-1 = linear)
  int* s_rot = reinterpret_cast<int*>(s_si + kDecMaxSeqs);
  volatile int* abort = reinterpret_cast<volatile int*>(s_rot + kDecMaxSeqs);

  const int lane = threadIdx.x & 31;
  const int b0 = blockIdx.x;
  const int nq = b0 < B ? (B - b0 + Gm.ctas - 1) / Gm.ctas : 0;
  const bool report = blockIdx.y == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncw);
    }
    *abort = 0;
    mbar_init_fence();
  }
  const int row_part = (W - 1) * row_bytes;  // the state part of a stage
  // sequences whose state rows are requested before the dependency wait
  // (at most one per ring stage: sequence q < NS goes to stage q; none in
  // the withheld-copy test mode, whose stages all take the normal path)
  const int n_pre = (W > 1 && Gm.state_early && !Gm.withhold_first)
                        ? min(min(nq, NS), SCONV_DECODE_EARLY_STAGES)
                        : 0;
  int issued0 = 0;  // (thread 0) stages already issued in full by the early fetch
  if (Gm.state_early) {
    // The caller promises that the previous kernel in the stream writes
    // none of this call's inputs but k and v: thread 0 requests the state
    // rows of the CTA's first n_pre sequences at once, waits for that
    // kernel, and then requests their K/V rows -- so every stage it has
    // started is complete (all its copies issued) before any wait that can
    // give up, and the drain below sees every copy in flight.
    if (threadIdx.x == 0) {
      unsigned ok = 0;  // bit q: sequence q's state index is valid
      for (int q = 0; q < n_pre; ++q) {
        const int64_t b = b0 + static_cast<int64_t>(q) * Gm.ctas;
        const int64_t si = P.state_indices ? static_cast<int64_t>(P.state_indices[b]) : b;
        if (si < 0 || si >= P.pool || (state_pos && state_pos[b] < 0)) continue;
        ok |= 1u << q;
        mbar_arrive_expect_tx(&full[q], static_cast<uint32_t>(stage_bytes));
        unsigned char* dst = ring + static_cast<size_t>(q) * stage_bytes;
        const uint16_t* sp = P.state + si * (W - 1) * srow;
        if (full_slice) {
          bulk_g2s(dst, sp, row_part, &full[q]);
        } else {
          for (int r = 0; r < W - 1; ++r) {
            if (kn) bulk_g2s(dst + r * row_bytes, sp + r * srow + g0 * 8, kn * 16, &full[q]);
            if (vn)
              bulk_g2s(dst + r * row_bytes + kn * 16, sp + r * srow + P.C + (vg0 - half) * 8,
                       vn * 16, &full[q]);
          }
        }
      }
      grid_dependency_wait();
      for (int q = 0; q < n_pre; ++q) {
        if (!(ok & (1u << q))) {
          mbar_arrive(&full[q]);  // skipped sequence: an empty phase
          continue;
        }
        const int64_t b = b0 + static_cast<int64_t>(q) * Gm.ctas;
        unsigned char* xd = ring + static_cast<size_t>(q) * stage_bytes + row_part;
        if (kn) bulk_g2s(xd, P.k + b * P.row_stride + g0 * 8, kn * 16, &full[q]);
        if (vn)
          bulk_g2s(xd + kn * 16, P.v + b * P.row_stride + (vg0 - half) * 8, vn * 16, &full[q]);
      }
      issued0 = n_pre;
    }
  } else {
    grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  }
  for (int q = threadIdx.x; q < nq; q += blockDim.x) {
    const int64_t b = b0 + static_cast<int64_t>(q) * Gm.ctas;
    int64_t si = b;
    int rot = -1;
    if (W > 1) {
      si = P.state_indices ? static_cast<int64_t>(P.state_indices[b]) : b;
      const int64_t pos = state_pos ? state_pos[b] : 0;
      if (si < 0 || si >= P.pool || pos < 0) {
        if (report) raise_flag(P.err, kFlagStateIndex);
        si = -1;
      }
      if (state_pos) rot = static_cast<int>(pos % (W - 1));
    }
    s_si[q] = si;
    s_rot[q] = rot;
    s_off[q] = slot_row_offset(P, P.slots[b], report);
  }
  if (nq == 0) return;

  // ---- producer (thread 0): sequence q (pool row si, -1 = skip) -> stage q % NS
  auto issue = [&](int q, long long si) {
    if (q == 0 && Gm.withhold_first) return;  // nothing will complete this stage
    const int st = q % NS;
    const int64_t b = b0 + static_cast<int64_t>(q) * Gm.ctas;
    if (si < 0) {
      mbar_arrive(&full[st]);  // skipped sequence: an empty phase
      return;
    }
    mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(stage_bytes));
    unsigned char* dst = ring + static_cast<size_t>(st) * stage_bytes;
    if (W > 1) {
      const uint16_t* sp = P.state + si * (W - 1) * srow;
      if (full_slice) {
        bulk_g2s(dst, sp, (W - 1) * row_bytes, &full[st]);
      } else {
        for (int r = 0; r < W - 1; ++r) {
          if (kn) bulk_g2s(dst + r * row_bytes, sp + r * srow + g0 * 8, kn * 16, &full[st]);
          if (vn)
            bulk_g2s(dst + r * row_bytes + kn * 16, sp + r * srow + P.C + (vg0 - half) * 8,
                     vn * 16, &full[st]);
        }
      }
    }
    unsigned char* xd = dst + (W - 1) * row_bytes;
    if (kn) bulk_g2s(xd, P.k + b * P.row_stride + g0 * 8, kn * 16, &full[st]);
    if (vn) bulk_g2s(xd + kn * 16, P.v + b * P.row_stride + (vg0 - half) * 8, vn * 16, &full[st]);
  };
  // linear state: new rows 0..W-2 <- stage rows 1..W-1; ring state: the
  // new row (stage row W-1) <- into row rot, the slot of its position (the
  // window's oldest position, no longer needed), and nothing else moves
  auto write_state = [&](int q) {
    const long long si = s_si[q];
    const int rot = LV ? s_rot[q] : -1;
    const unsigned char* src = ring + static_cast<size_t>(q % NS) * stage_bytes +
                               (rot < 0 ? row_bytes : (W - 1) * row_bytes);
    uint16_t* sp = P.state + si * (W - 1) * srow + (rot < 0 ? 0 : rot * srow);
    const int nrow = rot < 0 ? W - 1 : 1;
    if (full_slice) {
      bulk_s2g(sp, src, nrow * row_bytes);
    } else {
      for (int r = 0; r < nrow; ++r) {
        if (kn) bulk_s2g(sp + r * srow + g0 * 8, src + r * row_bytes, kn * 16);
        if (vn)
          bulk_s2g(sp + r * srow + P.C + (vg0 - half) * 8, src + r * row_bytes + kn * 16,
                   vn * 16);
      }
    }
    bulk_commit();
  };
  int issued = issued0;
  auto drain = [&]() {  // after giving up: let issued loads land (bounded)
    for (int d = max(0, issued - NS); d < issued; ++d) {
      if (d == 0 && Gm.withhold_first) continue;  // never requested
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(&full[d % NS], (d / NS) & 1) && global_ns() - t0 < kDrainTimeoutNs) {
      }
    }
    bulk_wait_all();
  };
  // With identity state indices thread 0 knows every pool row at once and
  // starts the copies before the index tables are even complete; otherwise
  // it waits for the tables.
  // The first sequence is requested alone and the rest of the ring once it
  // has landed: requested together, the stages of all CTAs share the
  // bandwidth and every CTA's first stage lands only when nearly all have
  // (measured on B200: decode step 8.9 -> 8.2 us).
  const int first_fill = 1;
  const bool identity = (W == 1) || P.state_indices == nullptr;
  if (identity && threadIdx.x == 0)
    for (; issued < min(first_fill, nq); ++issued) {
      const int64_t b = b0 + static_cast<int64_t>(issued) * Gm.ctas;
      issue(issued, (W == 1 || b < P.pool) ? b : -1);
    }
  __syncthreads();
  if (!identity && threadIdx.x == 0)
    for (; issued < min(first_fill, nq); ++issued) issue(issued, s_si[issued]);
  if (threadIdx.x == 0 && issued == nq) allow_dependent_launch();

  // ---- consumers: this thread's 8 channels
  const int lg = threadIdx.x;
  const bool active = lg < cs;
  const int g = g0 + (active ? lg : 0);
  const bool isv = g >= half;
  const int c0 = (isv ? g - half : g) * 8;
  const int d0 = c0 % D;
  uint16_t* cache = MX ? nullptr : (isv ? P.v_cache : P.k_cache) + (c0 / D) * P.stride_head + d0;
  const int64_t head_off = (c0 / D) * P.stride_head + d0;
  uint8_t* mxdata = MX ? (isv ? P.v_data : P.k_data) + head_off : nullptr;
  uint8_t* mxscale = MX ? (isv ? P.v_scale : P.k_scale) + (head_off >> 5) : nullptr;
  // taps kept packed (bf16) and widened at use: one token per sequence
  // makes the extra unpacking cheap, and the saved registers buy occupancy
  const uint16_t* w = (isv ? P.w_v : P.w_k) + c0;
  uint4 twp[W];
#pragma unroll
  for (int j = 0; j < W; ++j) twp[j] = ld_ro(w + static_cast<int64_t>(j) * P.C);
  const float* gam = (isv ? P.gamma_v : P.gamma_k) + (c0 / D) * gamma_hs + d0;  // per sequence

  for (int q = 0; q < nq; ++q) {
    const int st = q % NS;
    // a wait that gives up ends the whole warp at once; thread 0 first lets
    // its issued copies land
    if (!__all_sync(kFullMask, mbar_wait(&full[st], (q / NS) & 1, abort, Gm.timeout_ns))) {
      if (lane == 0) raise_flag(P.err, kFlagTimeout);
      if (threadIdx.x == 0) drain();
      return;
    }
    if (q == 0 && threadIdx.x == 0 && issued < nq) {
      for (; issued < min(NS, nq); ++issued) issue(issued, s_si[issued]);
      if (issued == nq) allow_dependent_launch();
    }
    const bool run = s_si[q] >= 0;
    if (run) {
      if (W > 1 && threadIdx.x == 0) write_state(q);
      // inactive lanes read column 0 and never store
      const unsigned char* stage =
          ring + static_cast<size_t>(st) * stage_bytes + (active ? lg : 0) * 16;
      float2 acc[4];
      // ring state: tap j reads row (rot + j) mod (W-1)
      const int rot = (LV && W > 1) ? max(s_rot[q], 0) : 0;
#pragma unroll
      for (int j = 0; j < W; ++j) {
        float2 rf[4], tw[4];
        const int row = j == W - 1 ? j : (rot + j < W - 1 ? rot + j : rot + j - (W - 1));
        unpack8(*reinterpret_cast<const uint4*>(stage + row * row_bytes), rf);
        unpack8(twp[j], tw);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = j == 0 ? fmul2(tw[e], rf[e]) : ffma2(tw[e], rf[e], acc[e]);
      }
      float2 s2 = fmul2(acc[0], acc[0]);
      s2 = ffma2(acc[1], acc[1], s2);
      s2 = ffma2(acc[2], acc[2], s2);
      s2 = ffma2(acc[3], acc[3], s2);
      const float ss = group_sum<G>(s2.x + s2.y);
      const float rn = rsqrt_approx(fmaf(ss, P.inv_d, P.eps));
      const long long off = s_off[q];
      if constexpr (MX) {
        // all lanes take part (the block scale is a 4-lane reduction)
        const float4 ga = __ldg(reinterpret_cast<const float4*>(gam));
        const float4 gb = __ldg(reinterpret_cast<const float4*>(gam) + 1);
        const float2 t[4] = {fmul2(acc[0], make_float2(ga.x, ga.y)),
                             fmul2(acc[1], make_float2(ga.z, ga.w)),
                             fmul2(acc[2], make_float2(gb.x, gb.y)),
                             fmul2(acc[3], make_float2(gb.z, gb.w))};
        mx_store8(t, rn, active && off >= 0, mxdata + (off >= 0 ? off : 0),
                  mxscale + (off >= 0 ? (off >> 5) : 0));
      } else if (active && off >= 0) {
        const float4 ga = __ldg(reinterpret_cast<const float4*>(gam));
        const float4 gb = __ldg(reinterpret_cast<const float4*>(gam) + 1);
        const float2 gm[4] = {make_float2(ga.x, ga.y), make_float2(ga.z, ga.w),
                              make_float2(gb.x, gb.y), make_float2(gb.z, gb.w)};
        const float2 rr = make_float2(rn, rn);
        uint4 o;
        o.x = pack_bf16x2(fmul2(fmul2(acc[0], rr), gm[0]));
        o.y = pack_bf16x2(fmul2(fmul2(acc[1], rr), gm[1]));
        o.z = pack_bf16x2(fmul2(fmul2(acc[2], rr), gm[2]));
        o.w = pack_bf16x2(fmul2(fmul2(acc[3], rr), gm[3]));
        st_stream(cache + off, o);
      }
    }
    __syncwarp();
    if (lane == 0) {
      if (threadIdx.x == 0 && run && W > 1) bulk_wait_read();  // write-back has read the stage
      mbar_arrive(&empty[st]);
    }
    bool gave_up = false;
    if (threadIdx.x == 0 && q >= 1 && issued < nq) {
      if (mbar_wait(&empty[(q - 1) % NS], ((q - 1) / NS) & 1, abort, Gm.timeout_ns)) {
        issue(issued, s_si[issued]);
        if (++issued == nq) allow_dependent_launch();
      } else {
        gave_up = true;
      }
    }
    if (__any_sync(kFullMask, gave_up)) {  // warp 0 leaves together
      if (lane == 0) raise_flag(P.err, kFlagTimeout);
      if (threadIdx.x == 0) drain();
      return;
    }
  }
  // the CTA may exit once its write-backs have read shared memory; the
  // global writes complete with the kernel
  if (threadIdx.x == 0) bulk_wait_read();
}

}  // namespace sconv
