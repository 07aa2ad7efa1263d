"""The ncu CSV summariser used for the profile notes (CPU only, on a small hand-written log)."""
import textwrap

from layer_streamed_qlora_streaming_b200 import ncu_summary

LOG = textwrap.dedent('''\
    ==PROF== Connected to process 1
    "ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
    "0","1","p","h","lst::<unnamed>::k_embed(int)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","us","2"
    "1","1","p","h","void lst::<unnamed>::k_gemm<256, 0, 0>(x)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","us","300"
    "2","1","p","h","void at::vectorized_elementwise_kernel<4>(x)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","us","50"
    "3","1","p","h","void lst::<unnamed>::k_gemm<256, 0, 0>(x)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","ms","0.1"
    "4","1","p","h","lst::<unnamed>::k_dequant(x)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","ns","98000"
    "5","1","p","h","lst::<unnamed>::k_embed(int)","1","7","(1,1,1)","(1,1,1)","0","10.0","s","gpu__time_duration.sum","us","2"
    ''')

TRAFFIC = textwrap.dedent('''\
    "ID","Kernel Name","Metric Name","Metric Unit","Metric Value"
    "0","k_gemm","dram__bytes_read.sum","Mbyte","300"
    "0","k_gemm","dram__bytes_write.sum","Mbyte","100"
    "0","k_gemm","gpu__time_duration.sum","us","200"
    "1","k_gemm","dram__bytes_read.sum","Gbyte","0.1"
    "1","k_gemm","dram__bytes_write.sum","Kbyte","500"
    "1","k_gemm","gpu__time_duration.sum","us","100"
    ''')


def test_step_table(tmp_path):
    p = tmp_path / "launches.csv"
    p.write_text(LOG)
    out = ncu_summary.step_table(str(p))
    assert out.startswith("total 0.50 ms over 4 launches")    # the torch kernel is left out
    assert "| `k_gemm<256, 0, 0>` | 2 | 0.40 | 80.0% |" in out
    assert "| `k_dequant` | 1 | 0.10 | 19.6% |" in out
    assert "| `k_embed` | 1 | 0.00 | 0.4% |" in out


def test_traffic_table(tmp_path):
    p = tmp_path / "traffic.csv"
    p.write_text(TRAFFIC)
    out = ncu_summary.traffic_table(str(p))
    assert "| dram__bytes_read.sum | 0.40 GB | 200.0 MB |" in out
    assert "| read + write | 0.50 GB | 250.2 MB |" in out
    assert "| gpu__time_duration.sum | 0.3 ms | 150 us |" in out
