/*
 * Test-only NVTX injection library: loaded by NVTX through
 * NVTX_INJECTION64_PATH, it records the domains created and every range
 * pushed (as "domain/name" lines) so a test can read them back with
 * nvtx_recorded().  Uses the public NVTX v3 callback interface.
 */
#include <nvtx3/nvToolsExt.h>   /* also brings the callback-table types */
#include <stdio.h>
#include <string.h>

static char g_log[1 << 16];
static size_t g_len = 0;
static char g_domains[16][64];
static int g_ndomains = 0;

static void append(const char* a, const char* b) {
  int n = snprintf(g_log + g_len, sizeof(g_log) - g_len, "%s/%s\n", a, b);
  if (n > 0 && g_len + (size_t)n < sizeof(g_log)) g_len += (size_t)n;
}

static nvtxDomainHandle_t NVTX_API domain_create(const char* name) {
  if (g_ndomains >= 16) return (nvtxDomainHandle_t)0;
  snprintf(g_domains[g_ndomains], sizeof(g_domains[0]), "%s", name);
  ++g_ndomains;
  return (nvtxDomainHandle_t)(size_t)g_ndomains;   /* 1-based index as the handle */
}

static int NVTX_API range_push(nvtxDomainHandle_t d, const nvtxEventAttributes_t* a) {
  size_t i = (size_t)d;
  const char* dom = (i >= 1 && i <= (size_t)g_ndomains) ? g_domains[i - 1] : "?";
  append(dom, (a && a->messageType == NVTX_MESSAGE_TYPE_ASCII && a->message.ascii) ? a->message.ascii : "?");
  return 0;
}

static int NVTX_API range_pop(nvtxDomainHandle_t d) {
  (void)d;
  return 0;
}

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE2, &table, &size)) return 0;
  if (size <= NVTX_CBID_CORE2_DomainCreateA) return 0;
  *table[NVTX_CBID_CORE2_DomainCreateA] = (NvtxFunctionPointer)domain_create;
  *table[NVTX_CBID_CORE2_DomainRangePushEx] = (NvtxFunctionPointer)range_push;
  *table[NVTX_CBID_CORE2_DomainRangePop] = (NvtxFunctionPointer)range_pop;
  return 1;
}

const char* nvtx_recorded(void) {
  g_log[g_len] = 0;
  return g_log;
}
