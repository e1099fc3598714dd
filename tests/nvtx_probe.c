/* An NVTX tool for tests/test_nvtx.py: records the name of every range pushed
 * in the process, and every pop, in a buffer the test reads back through
 * nvtx_probe_log().  The NVTX v3 loader inside libdit.so loads it from
 * NVTX_INJECTION64_PATH at the first NVTX call and calls
 * InitializeInjectionNvtx2, which installs the two handlers in the core
 * module's function table. */
#include <string.h>

#include <nvtx3/nvToolsExt.h>

static char log_buf[8192];
static size_t log_len;

static void add_line(const char* s) {
  const size_t n = strlen(s);
  if (log_len + n + 2 >= sizeof log_buf) return;
  memcpy(log_buf + log_len, s, n);
  log_len += n;
  log_buf[log_len++] = '\n';
  log_buf[log_len] = 0;
}

static int NVTX_API probe_push_a(const char* message) {
  add_line(message ? message : "(null)");
  return 0;
}

static int NVTX_API probe_pop(void) {
  add_line("pop");
  return 0;
}

const char* nvtx_probe_log(void) { return log_buf; }

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_export_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_export_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size) || size <= NVTX_CBID_CORE_RangePop)
    return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)probe_push_a;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)probe_pop;
  return 1;
}
