#include "profile.h"

namespace mo {

thread_local Profiler* g_prof = nullptr;

ProfScope::ProfScope(int kind, cudaStream_t stream, double flops) : s(stream) {
  Profiler* p = g_prof;
  if (p == nullptr || p->failed) return;
  if (p->used == p->recs.size()) {
    ProfRec r;
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
      p->failed = true;
      return;
    }
    p->recs.push_back(r);
  }
  rec = &p->recs[p->used++];
  rec->kind = kind;
  rec->flops = flops;
  if (cudaEventRecord(rec->a, s) != cudaSuccess) p->failed = true;
}

ProfScope::~ProfScope() {
  if (rec != nullptr && cudaEventRecord(rec->b, s) != cudaSuccess && g_prof) g_prof->failed = true;
}

}  // namespace mo
