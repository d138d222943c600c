/* A minimal NVTX tool library for tests: it records every range push and pop.
 *
 * An application that uses the NVTX v3 headers loads the library named by
 * NVTX_INJECTION64_PATH on its first NVTX call and calls its exported
 * InitializeInjectionNvtx2, which receives the export-table getter.  This one
 * asks for the callbacks table, fetches the core module's function table and
 * points RangePushA and RangePop at the recorders below.  A test reads the log
 * back through rec_log() / rec_depth() after loading this same file with
 * ctypes (dlopen of one path yields one handle, so the state is shared).
 */
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

static char g_log[65536];
static size_t g_len;
static int g_depth;

static void append(const char* s) {
  size_t n = strlen(s);
  if (g_len + n + 1 < sizeof(g_log)) {
    memcpy(g_log + g_len, s, n);
    g_len += n;
    g_log[g_len] = 0;
  }
}

static int rec_push(const char* name) {
  append("push ");
  append(name ? name : "(null)");
  append("\n");
  return g_depth++;
}

static int rec_pop(void) {
  append("pop\n");
  return --g_depth;
}

__attribute__((visibility("default"))) const char* rec_log(void) { return g_log; }
__attribute__((visibility("default"))) int rec_depth(void) { return g_depth; }
__attribute__((visibility("default"))) void rec_clear(void) {
  g_len = 0;
  g_log[0] = 0;
}

__attribute__((visibility("default"))) int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  if (!cb || cb->struct_size < sizeof(NvtxExportTableCallbacks)) return 0;
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size) || !table) return 0;
  if (size <= NVTX_CBID_CORE_RangePop) return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)rec_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)rec_pop;
  return 1;
}
