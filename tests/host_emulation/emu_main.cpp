// Runs attend_lean_kernel on host threads (one std::thread per CUDA thread, one cluster of
// CS x 256 threads per tile) over inputs read from a case directory, and writes its
// outputs back there.  Test infrastructure: it checks the kernel's control flow (every
// barrier and warp collective reached by the threads that must reach it), its memory
// accesses (with AddressSanitizer) and its results, without a GPU.
//
// usage: emu_lean <case dir>
//   <dir>/params.txt  key value lines (scalars), "row_off"/"slots" lines (kMaxLevels+1 ints) and
//                     an optional "seq_len" line (one length per sequence)
//   <dir>/{k_tok,v_tok,k_node,v_node,q}.bin  bf16 arrays in the library's layouts
//   writes <dir>/{out,sel,entries}.bin and <dir>/err.txt (the workspace error word)
#include <fstream>
#include <map>
#include <sstream>
#include <thread>

#include "lean_extracted.h"

namespace emu {
thread_local int t_tid, t_block, t_crank, t_cs, t_grid = 1;
int g_nt = 256;
std::vector<uint32_t> g_cta_pred;
thread_local long t_cluster_gen = -1;
thread_local unsigned char *t_smem;
std::vector<unsigned char *> g_cluster_smem;
size_t g_smem_bytes;
std::vector<TBarrier> g_cta_bar;
TBarrier g_cluster_bar;
std::vector<TBarrier> g_warp_bar;
std::vector<uint32_t> g_warp_slot;
std::vector<Where> g_where;
int g_cs = 0;

void report_and_abort(const char *why) {
  static std::mutex m;
  std::lock_guard<std::mutex> lk(m);
  fprintf(stderr, "STALL: %s\n", why);
  std::vector<std::pair<std::string, int>> seen;  // where the threads wait
  for (int r = 0; r < g_cs; ++r)
    for (int t = 0; t < 256; ++t) {
      char buf[128];
      snprintf(buf, sizeof buf, "rank %d %s:%d", r, (const char *)g_where[r * 256 + t].what,
               (int)g_where[r * 256 + t].line);
      bool f = false;
      for (auto &s : seen)
        if (s.first == buf) {
          s.second++;
          f = true;
        }
      if (!f) seen.push_back({buf, 1});
    }
  for (auto &s : seen) fprintf(stderr, "  %-40s threads %d\n", s.first.c_str(), s.second);
  fflush(stderr);
  _exit(3);
}
}  // namespace emu

using namespace recsa;

template <int G, int CS, int RPH>
void run_cluster(const AttendArgs &a, int tile, size_t smem_bytes) {
  using namespace emu;
  g_cs = CS;
  g_smem_bytes = smem_bytes;
  std::vector<std::vector<unsigned char>> sm(CS, std::vector<unsigned char>(smem_bytes, 0xAB));
  g_cluster_smem.assign(CS, nullptr);
  for (int r = 0; r < CS; ++r) g_cluster_smem[r] = sm[r].data();
  g_cta_bar = std::vector<TBarrier>(CS);
  for (int r = 0; r < CS; ++r) g_cta_bar[r].init(256, "syncthreads");
  g_cluster_bar.init(256 * CS, "cluster");
  g_warp_bar = std::vector<TBarrier>(CS * 8);
  for (auto &w : g_warp_bar) w.init(32, "warp");
  g_warp_slot.assign(CS * 8 * 32, 0);
  g_where = std::vector<Where>(CS * 256);
  std::vector<std::thread> th;
  for (int r = 0; r < CS; ++r)
    for (int t = 0; t < 256; ++t)
      th.emplace_back([&, r, t] {
        t_tid = t;
        t_crank = r;
        t_cs = CS;
        t_block = tile * CS + r;
        t_smem = g_cluster_smem[r];
        attend_lean_kernel<G, CS, RPH>(a);
        g_where[r * 256 + t].line = -1;
        g_where[r * 256 + t].what = "exited";
      });
  for (auto &x : th) x.join();
}

template <typename T>
std::vector<T> read_bin(const std::string &path) {
  std::ifstream f(path, std::ios::binary | std::ios::ate);
  if (!f) {
    fprintf(stderr, "cannot read %s\n", path.c_str());
    exit(2);
  }
  const size_t n = (size_t)f.tellg();
  std::vector<T> v(n / sizeof(T) + 1);  // one spare element: an empty file still has a pointer
  f.seekg(0);
  f.read(reinterpret_cast<char *>(v.data()), (std::streamsize)n);
  v.resize(std::max<size_t>(n / sizeof(T), 1));
  return v;
}
template <typename T>
void write_bin(const std::string &path, const std::vector<T> &v) {
  std::ofstream f(path, std::ios::binary);
  f.write(reinterpret_cast<const char *>(v.data()), (std::streamsize)(v.size() * sizeof(T)));
}

int main(int argc, char **argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: emu_lean <case dir>\n");
    return 2;
  }
  const std::string dir = argv[1];
  std::map<std::string, double> kv;
  std::vector<int64_t> row_off, slots, seq_len;
  {
    std::ifstream f(dir + "/params.txt");
    std::string line;
    while (std::getline(f, line)) {
      std::istringstream ss(line);
      std::string key;
      ss >> key;
      if (key == "row_off" || key == "slots" || key == "seq_len") {
        int64_t x;
        auto &dst = key == "row_off" ? row_off : key == "slots" ? slots : seq_len;
        while (ss >> x) dst.push_back(x);
      } else {
        double x;
        ss >> x;
        kv[key] = x;
      }
    }
  }
  const int G = (int)kv["G"], CS = (int)kv["CS"], RPH = (int)kv["RPH"];
  auto ktok = read_bin<uint16_t>(dir + "/k_tok.bin"), vtok = read_bin<uint16_t>(dir + "/v_tok.bin");
  auto knode = read_bin<uint16_t>(dir + "/k_node.bin"), vnode = read_bin<uint16_t>(dir + "/v_node.bin");
  auto q = read_bin<uint16_t>(dir + "/q.bin");

  // RoPE table as the library's workspace holds it: cos/sin in fp64, stored fp32, the pair
  // of frequencies (2u, 2u+1) as (cos, cos', sin, sin')
  const int table_rows = (int)kv["table_rows"];
  const double base = kv["rope_base"];
  std::vector<unsigned char> ws(kWsHeader + (size_t)table_rows * kHalf * 8, 0);
  WsHeader *hdr = reinterpret_cast<WsHeader *>(ws.data());
  hdr->magic = kWsMagic;
  hdr->table_rows = table_rows;
  float *table = reinterpret_cast<float *>(ws.data() + kWsHeader);
  for (int pos = 0; pos < table_rows; ++pos)
    for (int i = 0; i < kHalf; ++i) {
      const double th = (double)pos * std::pow(base, -2.0 * i / kD);
      float *pair = table + (size_t)pos * 2 * kHalf + (i >> 1) * 4 + (i & 1);
      pair[0] = (float)std::cos(th);
      pair[2] = (float)std::sin(th);
    }

  const int tiles = (int)kv["tiles"], top_k = (int)kv["top_k"], sel_levels = (int)kv["sel_levels"];
  std::vector<float> out(q.size(), 0.f);
  std::vector<int32_t> sel((size_t)tiles * sel_levels * std::min(std::max(top_k, 1), 64), -7), ent((size_t)tiles * 2, 0);

  AttendArgs a = {};
  a.k_tok = ktok.data();
  a.v_tok = vtok.data();
  a.k_node = knode.data();
  a.v_node = vnode.data();
  a.q = q.data();
  a.out = out.data();
  a.hdr = hdr;
  a.table = reinterpret_cast<const float2 *>(table);
  a.sel_idx = (top_k >= 1 && top_k <= 64) ? sel.data() : nullptr;
  a.sel_levels = sel_levels;
  a.entries = ent.data();
  a.seq_len = seq_len.empty() ? nullptr : seq_len.data();
  a.cap = (int64_t)kv["cap"];
  a.length = (int64_t)kv["length"];
  for (int i = 0; i <= kMaxLevels; ++i) {
    a.row_off[i] = row_off.at(i);
    a.slots[i] = slots.at(i);
    int64_t sp = 1;
    for (int l = 0; l < i && sp <= ((int64_t)1 << 30); ++l) sp *= (int64_t)kv["b"];
    sp = std::min<int64_t>(sp, (int64_t)1 << 30 | 1);
    a.span[i] = (int32_t)sp;
    a.nlen[i] = (int32_t)((a.length + sp - 1) / sp);
  }
  a.levels = (int)kv["levels"];
  a.hkv = (int)kv["hkv"];
  a.hq = a.hkv * G;
  a.b = (int)kv["b"];
  a.top_k = top_k;
  a.nq = (int)kv["nq"];
  a.causal = (int)kv["causal"];
  a.out_fp32 = 1;
  a.table_rows_needed = (int)kv["table_rows_needed"];
  a.max_cand = (int)kv["max_cand"];
  a.scale = (float)kv["scale"];
  a.tiles = tiles;
  const LeanLayout Ls = lean_layout(G, CS, a.max_cand);
  for (int tile = 0; tile < tiles; ++tile) {
    bool ran = false;
#define RUN(g, cs, rph)                                   \
  if (G == g && CS == cs && RPH == rph) {                 \
    run_cluster<g, cs, rph>(a, tile, (size_t)Ls.total);   \
    ran = true;                                           \
  }
    RUN(1, 2, 4) RUN(2, 2, 4) RUN(4, 2, 4) RUN(1, 4, 2) RUN(2, 4, 2) RUN(4, 4, 2) RUN(8, 4, 2)
    RUN(1, 4, 3) RUN(2, 4, 3) RUN(4, 4, 3)
#undef RUN
    if (!ran) {
      fprintf(stderr, "no lean instance for G=%d CS=%d RPH=%d\n", G, CS, RPH);
      return 2;
    }
  }
  write_bin(dir + "/out.bin", out);
  write_bin(dir + "/sel.bin", sel);
  write_bin(dir + "/entries.bin", ent);
  std::ofstream(dir + "/err.txt") << hdr->err << "\n";
  return 0;
}
