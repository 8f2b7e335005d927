/*
 * A minimal NVTX tool for the tests: loaded by the NVTX runtime of any library
 * that emits ranges when NVTX_INJECTION64_PATH names this shared object. It
 * writes one line per range push ("push <name>") and pop ("pop") to the file
 * named by FLCE_NVTX_LOG. It uses only the documented injection interface of
 * the NVTX 3 headers (the callback export table and the core module's
 * function table).
 */
#include <nvtx3/nvToolsExt.h>
#include <stdio.h>
#include <stdlib.h>

static FILE* g_out = NULL;

static int record_push(const char* message) {
  if (g_out) {
    fprintf(g_out, "push %s\n", message ? message : "");
    fflush(g_out);
  }
  return 0;
}

static int record_pop(void) {
  if (g_out) {
    fputs("pop\n", g_out);
    fflush(g_out);
  }
  return 0;
}

__attribute__((visibility("default"))) int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  const char* path = getenv("FLCE_NVTX_LOG");
  if (!cb || !path || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size)) return 0;
  if (size <= NVTX_CBID_CORE_RangePop) return 0;
  g_out = fopen(path, "w");
  if (!g_out) return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)record_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)record_pop;
  return 1;
}
