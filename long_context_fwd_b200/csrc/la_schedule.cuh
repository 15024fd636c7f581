// la_schedule.cuh -- how the prefill kernel's (b, h) sequences become work
// items (host and device code: the host enumerates the same items in tests).
#pragma once
#include <cstdint>

namespace la {
namespace fwd {

#define LA_HD __host__ __device__ __forceinline__

constexpr int BLK = 128;  // tokens per block
constexpr int HD = 128;   // head dimension (D = E)

template <class T>
LA_HD T la_min(T a, T b) { return a < b ? a : b; }
template <class T>
LA_HD T la_max(T a, T b) { return a < b ? b : a; }

struct Params {
  const float* slopes;        // [H]
  float* prefix;              // [nseq][2][HD*HD] inclusive chunk states (chunked runs)
  unsigned long long* flags;  // publication flags: the chunk scan's chunk numbers (zeroed
                              // before the launch) or this launch's tag (hand-over, split scan)
  int* ticket;                // work counter (chunk scan), zeroed before the launch
  unsigned long long tag;     // nonzero and unique to the launch: the flag value the hand-over
                              // and the split scan publish, so their flags need no zeroing
  const float* init_state;    // nullable [nseq][HD*HD]
  float* final_state;         // nullable [nseq][HD*HD]
  int* status;                // sticky error word
  int H, N, nseq, L, nchunks, total;
  int ticket_base;            // first ticket handed out (0 except in fault-injection runs)
  int mode;                   // work items: MODE_TICKETS, MODE_HANDOVER or MODE_SPLIT_SCAN
  int state_only;             // the state pass alone (lightning_attn_state): every chunk a
                              // local-state item, no outputs; the last writes final_state
  int nblk;                   // 128-token blocks per sequence
  int F, G2;                  // split scan: blocks of each sequence in the local-state pass;
                              // CTAs whose outputs cover that part
  long long P;                // split scan: nseq * F
  int cslot[4];               // q, k, v, out tensor maps: where t, h, b sit (make_tmap_4d)
  int D, E;                   // the caller's head dimensions (64 or 128; tiles are 128 wide,
                              // the tensor maps zero-fill the columns past D or E)
  float* out;                 // the output and its element strides {b, h, t}, for rows that
  long long ostride[3];       // are stored without TMA (anti-causal runs, first block)
  const uint16_t* gate;       // fused layer: bf16 gate (before the sigmoid), element
  long long gstride[3];       // strides {b, h, t}, e contiguous
  const float* norm_w;        // fused layer: RMSNorm weight [H][E]
  float eps;                  // fused layer: RMSNorm epsilon
  unsigned long long wait_limit_ns;
  // Two operators in one launch (paired = 1): CTA 2j + r computes role r of
  // virtual CTA j (role 1 takes the second set of tensor maps and these
  // pointers), so both roles of a pair read shared operands close in time.
  int paired;
  int* ticket1;
  unsigned long long* flags1;
  float* prefix1;
  float* out1;
};

// How sequences become work items (chosen on the host):
//  MODE_TICKETS     whole sequences (static stride) or, with chunks, the parallel
//                   chunk scan handed out by an atomic ticket;
//  MODE_HANDOVER    at least as many sequences as CTAs: equal shares of blocks,
//                   a sequence crossing a share boundary handed over through its
//                   final state;
//  MODE_SPLIT_SCAN  fewer sequences than CTAs: a local-state pass over the first
//                   part of every sequence shared equally by all CTAs, then equal
//                   shares of output blocks, entering states chained from the
//                   published local states.
constexpr int MODE_TICKETS = 0, MODE_HANDOVER = 1, MODE_SPLIT_SCAN = 2;

struct Item {
  int seq, chunk, t0, Lc, nb;
  bool phase1;   // local state first, published before the outputs (parallel scan)
  bool p2;       // outputs (false: a local-state-only item of the split scan)
  bool publish;  // final state published after the outputs (balanced split)
  bool enter;    // starts from a published state: prefix[enter_slot] once flags[enter_slot] == enter_val
  bool last;     // ends its sequence (final state goes to the caller)
  int enter_slot, pub_slot;
  unsigned long long enter_val, pub_val;
};

// Ticket w of a chunked or unchunked run: chunk-major order, so every chunk of
// a sequence is handed out after its predecessor.
LA_HD Item decode_item(const Params& p, int w) {
  Item it;
  it.chunk = w / p.nseq;
  it.seq = w - it.chunk * p.nseq;
  it.t0 = it.chunk * p.L;
  it.Lc = la_min(p.L, p.N - it.t0);
  it.nb = (it.Lc + BLK - 1) / BLK;
  it.phase1 = p.state_only || it.chunk + 1 < p.nchunks;
  it.p2 = !p.state_only;
  it.publish = false;
  it.enter = it.chunk > 0;
  it.last = it.chunk + 1 == p.nchunks;
  it.enter_slot = it.seq * 2 + ((it.chunk - 1) & 1);
  it.enter_val = static_cast<unsigned long long>(it.chunk);
  it.pub_slot = it.seq * 2 + (it.chunk & 1);
  it.pub_val = static_cast<unsigned long long>(it.chunk) + 1u;
  return it;
}

// Balanced split (at least as many sequences as CTAs): CTA j owns blocks
// [j*T/G, (j+1)*T/G) of the concatenation of all sequences' 128-token blocks
// (T blocks, G CTAs), at least one whole sequence's worth.  So at most one
// sequence crosses each CTA boundary: CTA j computes that sequence's first part
// FIRST and publishes its final state in slot j; CTA j+1 computes the rest LAST,
// starting from slot j, which by then has long been written.  Item k of this CTA:
// the first part (if any), the whole sequences in order, then the rest of the
// sequence that CTA j-1 began (if any).
// The CTA's split, computed once at launch into misc[4..9]: head sequence and
// its length in blocks (0: none), first whole sequence and their count, tail
// sequence and its first block (0: none).
LA_HD void balanced_split(const Params& p, int64_t G, int64_t j, volatile uint32_t* m) {
  const int64_t nblk = (p.N + BLK - 1) / BLK;
  const int64_t T = nblk * p.nseq;
  const int64_t b0 = T * j / G, b1 = T * (j + 1) / G;
  const int64_t s_first = b0 / nblk, s_last = (b1 - 1) / nblk;
  const int64_t tail_b0 = b0 - s_first * nblk;          // > 0: continues CTA j-1's sequence
  const int64_t head_len = b1 < (s_last + 1) * nblk ? b1 - s_last * nblk : 0;
  const int64_t full0 = s_first + (tail_b0 ? 1 : 0), full1 = s_last + (head_len ? 0 : 1);
  m[4] = static_cast<uint32_t>(s_last);
  m[5] = static_cast<uint32_t>(head_len);
  m[6] = static_cast<uint32_t>(full0);
  m[7] = static_cast<uint32_t>(full1 > full0 ? full1 - full0 : 0);
  m[8] = static_cast<uint32_t>(s_first);
  m[9] = static_cast<uint32_t>(tail_b0);
}

LA_HD bool balanced_item(const Params& p, int j, const volatile uint32_t* m, int k, Item& it) {
  const int nblk = (p.N + BLK - 1) / BLK;
  const int head_len = static_cast<int>(m[5]), nfull = static_cast<int>(m[7]);
  const int tail_b0 = static_cast<int>(m[9]);
  int seq, blk0 = 0, blk1 = nblk;
  it.phase1 = false;
  it.p2 = true;
  it.publish = it.enter = false;
  it.enter_slot = j - 1;
  it.pub_slot = j;
  it.enter_val = it.pub_val = p.tag;
  int i = k;
  if (head_len && i == 0) {
    seq = static_cast<int>(m[4]);
    blk1 = head_len;
    it.publish = true;
  } else {
    if (head_len) --i;
    if (i < nfull) {
      seq = static_cast<int>(m[6]) + i;
    } else if (tail_b0 && i == nfull) {
      seq = static_cast<int>(m[8]);
      blk0 = tail_b0;
      it.enter = true;
    } else {
      return false;
    }
  }
  it.seq = seq;
  it.chunk = it.enter ? 1 : 0;
  it.t0 = blk0 * BLK;
  it.Lc = la_min(blk1 * BLK, p.N) - it.t0;
  it.nb = blk1 - blk0;
  it.last = !it.publish;
  return true;
}

// Split scan.  The local-state pass runs over the stream made of the first F
// blocks of every sequence, concatenated (P = nseq * F blocks).  The stream is
// cut at three kinds of boundaries: the CTAs' equal shares of this pass,
// A_i = floor(P i / G); the starts of the G2 = G - nseq output shares that
// cover the same blocks, R_k = floor(P k / G2); and the sequence starts s F.
// Each piece between consecutive boundaries is a local-state item; piece
// [x, y) publishes the state sum_{t in [x,y)} gamma^(y*128-1-t) k_t^T v_t in
// slot s1_slot(x).  The other nseq CTAs each compute the last nblk - F blocks
// of one sequence.  An output share that starts at stream position X inside
// sequence s chains the pieces of [s F, X): X is always a boundary, so no
// piece straddles it.  Shares of both passes are equal, so no CTA waits long.
LA_HD int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// End of the piece that starts at stream position x.
LA_HD int64_t s1_next(const Params& p, int64_t G, int64_t x) {
  const int64_t G2 = p.G2;
  const int64_t ia = cdiv64((x + 1) * G, p.P);  // first pass share starting after x
  const int64_t a = ia < G ? p.P * ia / G : p.P;
  const int64_t kr = cdiv64((x + 1) * G2, p.P);  // first output share starting after x
  const int64_t r = kr < G2 ? p.P * kr / G2 : p.P;
  const int64_t sq = (x / p.F + 1) * p.F;        // next sequence start
  return la_min(la_min(a, r), la_min(sq, static_cast<int64_t>(p.P)));
}

// Slot of the piece that starts at stream position x: the number of
// boundaries at or before x, counting coincident ones separately (strictly
// increasing over piece starts; below 2G).
LA_HD int s1_slot(const Params& p, int64_t G, int64_t x) {
  const int64_t G2 = p.G2;
  const int64_t na = la_min(G, cdiv64((x + 1) * G, p.P));
  const int64_t nr = la_min(G2, cdiv64((x + 1) * G2, p.P)) - 1;
  const int64_t ns = x / p.F;
  return static_cast<int>(na + nr + ns - 1);
}

// This CTA's split-scan work, computed once at launch into misc: [4] number of
// local-state items n1 (at most 4: a pass share is shorter than an output
// share and than a sequence's first part, so at most two output-share starts
// and one sequence start fall inside it); [5..5+n1] their stream boundaries;
// [11..11+n1) their slots; [16], [17] this CTA's output share [r0, r1) of the
// stream (CTAs below G2).  Returns false if the bound were ever exceeded.
constexpr int SPLIT_MAX_PIECES = 5;
LA_HD bool split_scan_setup(const Params& p, int64_t G, int64_t i, volatile uint32_t* m) {
  const int64_t G2 = p.G2;
  const int64_t end = p.P * (i + 1) / G;
  int n = 0;
  int64_t x = p.P * i / G;
  m[5] = static_cast<uint32_t>(x);
  while (x < end) {
    if (n == SPLIT_MAX_PIECES) return false;
    m[11 + n] = static_cast<uint32_t>(s1_slot(p, G, x));
    x = s1_next(p, G, x);
    ++n;
    m[5 + n] = static_cast<uint32_t>(x);
  }
  m[4] = static_cast<uint32_t>(n);
  if (i < G2) {
    m[16] = static_cast<uint32_t>(p.P * i / G2);
    m[17] = static_cast<uint32_t>(i + 1 < G2 ? p.P * (i + 1) / G2 : p.P);
  }
  return true;
}

LA_HD bool split_scan_item(const Params& p, int i, const volatile uint32_t* m, int k, Item& it) {
  const int F = p.F;
  const int n1 = static_cast<int>(m[4]);
  int seq, blk0, blk1;
  it.publish = it.enter = it.last = false;
  it.pub_val = it.enter_val = p.tag;
  it.enter_slot = 0;
  if (k < n1) {  // local state of one piece of this CTA's pass share
    const int x = static_cast<int>(m[5 + k]), y = static_cast<int>(m[6 + k]);
    seq = x / F;
    blk0 = x - seq * F;
    blk1 = y - seq * F;
    it.phase1 = true;
    it.p2 = false;
    it.publish = true;
    it.pub_slot = static_cast<int>(m[11 + k]);
  } else {
    int k2 = k - n1;
    it.phase1 = false;
    it.p2 = true;
    it.pub_slot = 0;
    if (i < p.G2) {  // outputs of stream blocks [r0, r1), split at sequence starts
      const int r0 = static_cast<int>(m[16]), r1 = static_cast<int>(m[17]);
      if (r1 <= r0) return false;
      const int sa = r0 / F, sb = (r1 - 1) / F;
      if (k2 > sb - sa) return false;
      // in stream order: a first piece that needs an entering state starts
      // right after this CTA's local-state pass, when the pieces it chains
      // have just been published (still in L2) -- later, behind a stream of
      // output blocks, their loads took several times longer
      seq = sa + k2;
      blk0 = la_max(r0, seq * F) - seq * F;
      blk1 = la_min(r1, (seq + 1) * F) - seq * F;
      it.enter = blk0 > 0;
    } else {  // the last nblk - F blocks of sequence i - G2
      if (k2 > 0) return false;
      seq = i - p.G2;
      blk0 = F;
      blk1 = p.nblk;
      it.enter = true;
      it.last = true;
    }
  }
  it.seq = seq;
  it.chunk = it.enter ? 1 : 0;
  it.t0 = blk0 * BLK;
  it.Lc = la_min(blk1 * BLK, p.N) - it.t0;
  it.nb = blk1 - blk0;
  return true;
}

// Work item for work index w of CTA i (of G); false once the CTA has no more.
LA_HD bool get_item(const Params& p, int G, int i, const volatile uint32_t* m, int w, Item& it) {
  if (p.mode == MODE_HANDOVER) return balanced_item(p, i, m, w, it);
  if (p.mode == MODE_SPLIT_SCAN) return split_scan_item(p, i, m, w, it);
  if (w >= p.total) return false;
  it = decode_item(p, w);
  return true;
}

// This CTA's share of a static split, computed once at launch into m (shared
// memory on the GPU).  False only if a split-scan share broke its bound.
LA_HD bool setup_split(const Params& p, int G, int i, volatile uint32_t* m) {
  if (p.mode == MODE_HANDOVER) balanced_split(p, G, i, m);
  if (p.mode == MODE_SPLIT_SCAN) return split_scan_setup(p, G, i, m);
  return true;
}

}  // namespace fwd
}  // namespace la
