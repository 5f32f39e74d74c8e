// Host-buffer entry point: the whole path (stats -> routing -> select -> attention) on
// Q, K, V in host memory, with O written back to host memory, pipelined over ranges of
// (batch, head) pairs.
//
// Every step of the method is independent across (batch, head) pairs (PISA explainer,
// section 2: block statistics, selection and the fused attention are all per head), so
// the flattened [B*H, N, d] problem splits into `chunks` contiguous ranges. Range c
// lives in workspace slot c % kSlots. Three streams overlap the copies with the
// kernels:
//   copy-in stream:  H2D of range c (one cudaMemcpyAsync per tensor), after the slot's
//                    previous occupant (range c - kSlots) has been copied out;
//   caller's stream: the kernels of range c, after its copy-in;
//   copy-out stream: D2H of range c's output, after its kernels.
// The call returns when O holds the whole result (it synchronises all three).
#pragma once

#include <cstddef>
#include <vector>

namespace pisa_host {

constexpr int kSlots = 3;           // workspace slots (ranges in flight)
constexpr size_t kAlign = 256;      // every sub-buffer starts on a 256-byte boundary

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of one slot's buffers for ranges of up to R (batch, head) pairs.
struct SlotLayout {
  size_t q, k, v, o, kbar, s0, s1, hbar, m, idx, bytes;
};

inline SlotLayout slot_layout(int64_t R, int64_t N, int64_t d, int64_t nB, int64_t topk, int order, bool routed) {
  SlotLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  const size_t act = size_t(R) * N * d * 2;
  L.q = take(act);
  L.k = take(act);
  L.v = take(act);
  L.o = take(act);
  L.kbar = take(size_t(R) * nB * d * 4);
  L.s0 = take(size_t(R) * nB * d * 4);
  const bool per_block = order == PISA_ORDER_FIRST || routed;
  L.s1 = take(per_block ? size_t(R) * nB * d * d * 2 : (order == PISA_ORDER_HYBRID ? size_t(R) * d * d * 4 : 0));
  L.hbar = take(routed ? size_t(R) * d * d * 4 : 0);
  L.m = take(routed ? size_t(R) * nB * 4 : 0);
  L.idx = take(size_t(R) * nB * topk * 4);
  L.bytes = off;
  return L;
}

inline int64_t range_size(int64_t BH, int chunks) { return (BH + chunks - 1) / chunks; }

inline size_t workspace_bytes(const pisa_shape_t& s, int topk, int order, bool routed, int chunks) {
  const int64_t BH = int64_t(s.B) * s.H;
  const int c = int(chunks < BH ? chunks : BH);
  const int slots = c < kSlots ? c : kSlots;
  const int64_t nB = (int64_t(s.N) + s.block - 1) / s.block;
  return size_t(slots) * slot_layout(range_size(BH, c), s.N, s.d, nB, topk, order, routed).bytes;
}

}  // namespace pisa_host
