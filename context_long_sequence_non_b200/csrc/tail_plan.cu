// tail_plan.cu -- host-side planning of the tail split: which work items of an attention
// launch run as key ranges, and the workspace their partials need.  The kernel side (the
// 1-D grid form that runs the plan) is attn_sm100.cu; the fold is simt.cu's
// combine_tail_kernel.
#include <cstddef>

#include "kernels.h"

namespace cpattn {
namespace {

constexpr long long kItemRows = 256;  // query rows per work item (two 128-row Q tiles)
constexpr int kKeyBlock = 128;        // keys per K/V block

}  // namespace

// Candidate tail splits: the last rem + k * sms work items (k = 0: the partial last wave
// alone; k = 1: that wave and the whole wave before it) as p key ranges each, the rest
// whole.  p <= 8 for k = 0 and p <= 4 for k = 1, which bounds the workspace.
constexpr int kTailMaxParts[2] = {8, 4};

TailSplit tail_split_plan(int B, int H, int Sq, int Skv) {
  TailSplit t{};
  const long long pairs = (Sq + kItemRows - 1) / kItemRows;
  const long long items = pairs * H * B;
  const int sms = sm_count();
  const int n_kv = (Skv + kKeyBlock - 1) / kKeyBlock;
  if (items < 1 || items > 0x7fffffffLL || n_kv < 4) return t;
  const long long rem = items % sms;  // items of the last, partial wave
  if (rem == 0) return t;
  // Makespan in units of one whole item's time, each CTA paying a fixed cost (c) of about
  // eight key blocks -- start-up, Q load, pipeline fill, epilogue and its share of the
  // combine; calibrated on measured splits of short and long items: whole waves cost 1 + c,
  // and the split items' ranges run in ceil(tail * p / sms) short waves of 1/p + c.  Split
  // only when that saves at least 0.5 %.
  const double c = 8.0 / n_kv;
  const double whole = double((items + sms - 1) / sms) * (1.0 + c);
  double best = whole * 0.995;
  for (int k = 0; k < 2; ++k) {
    const long long tail = rem + (long long)k * sms;
    if (tail > items) break;
    const double before = double((items - tail) / sms) * (1.0 + c);
    for (int p = 2; p <= kTailMaxParts[k] && p <= n_kv / 2; ++p) {
      const long long short_waves = (tail * p + sms - 1) / sms;
      const double span = before + double(short_waves) * (1.0 / p + c);
      if (span < best) {
        best = span;
        t.n_full = int(items - tail);
        t.n_tail = int(tail);
        t.parts = p;
      }
    }
  }
  return t;
}

size_t tail_split_workspace_bound(int B, int H, int Sq, int D) {
  const long long pairs = (Sq + kItemRows - 1) / kItemRows;
  const long long items = pairs * H * B;
  const int sms = sm_count();
  if (items < 1 || items > 0x7fffffffLL || items % sms == 0) return 0;
  TailSplit t{};
  long long worst = 0;
  for (int k = 0; k < 2; ++k) {
    const long long tail = items % sms + (long long)k * sms;
    if (tail <= items && tail * kTailMaxParts[k] > worst) {
      worst = tail * kTailMaxParts[k];
      t.n_tail = int(tail);
      t.parts = kTailMaxParts[k];
    }
  }
  return tail_split_workspace(t, D);
}

size_t tail_split_workspace(const TailSplit& t, int D) {
  if (t.parts < 2) return 0;
  const size_t rows = size_t(t.parts) * t.n_tail * kItemRows;
  return ((rows * D * 4 + 255) & ~size_t(255)) + rows * 4;
}

}  // namespace cpattn
