// Planning and launch sequence of the SOAP path.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/mo.h"
#include "ns_plan.h"

namespace mo {

struct SoapItem {
  mo_soap_mat m;
  int32_t* flag = nullptr;
};

// SOAP-Muon: the Muon momentum (mu, Nesterov) is preconditioned in the
// previous bases, orthogonalised by Newton-Schulz (ns: steps, coefficients,
// eps, lr, weight decay, scale mode) and applied; the bases are refreshed
// afterwards for the next step.
struct SoapMuonExt {
  float mu = 0.95f;
  bool nesterov = true;
  NsCall ns;
};

void soap_workspace(const int64_t* rows, const int64_t* cols, int n, size_t* min_bytes, size_t* full_bytes);

// Exact workspace for these matrices (sides as given).
size_t soap_workspace_exact(const std::vector<SoapItem>& items, bool soap_muon = false);

// Enqueue one SOAP step for every item.  Planning errors set *err.
cudaError_t soap_run(const std::vector<SoapItem>& items, const mo_soap_cfg& cfg, int64_t step, char* ws,
                     size_t ws_bytes, cudaStream_t stream, std::string* err,
                     const SoapMuonExt* ext = nullptr);

}  // namespace mo
