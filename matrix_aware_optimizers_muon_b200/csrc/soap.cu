// SOAP driver (per-step power iteration + QR basis refresh).
#include "ns_plan.h"
#include "soap_plan.h"

namespace mo {

void soap_workspace(const int64_t* rows, const int64_t* cols, int n, size_t* min_bytes, size_t* full_bytes) {
  (void)rows; (void)cols; (void)n;
  *min_bytes = WS_HEADER;
  *full_bytes = WS_HEADER;
}

cudaError_t soap_run(const std::vector<SoapItem>& items, const mo_soap_cfg& cfg, int64_t step, char* ws,
                     size_t ws_bytes, cudaStream_t stream, std::string* err) {
  (void)items; (void)cfg; (void)step; (void)ws; (void)ws_bytes; (void)stream;
  *err = "the SOAP path is not built in this version";
  return cudaErrorNotSupported;
}

}  // namespace mo
